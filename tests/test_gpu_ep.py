"""The expert-parallel form of the layer on one GPU with N virtual ranks
(sigmoid_top_routing_warp_b200/ep.py: moe_ep_pack, the k = 1 expert layer
over received rows, moe_shared_expert, moe_combine; the all-to-alls are
device copies).  Each virtual rank's output is checked against the CPU
oracle's whole layer on its tokens (the bf16 bar) and must equal
moe_forward's on the same tokens bit for bit.  Multi-GPU runs of the same protocol (NCCL all-to-alls)
are not measured here: every call in this build has one GPU."""
import numpy as np
import pytest
import torch

from helpers import assert_close_bf16, oracle_cfg, oracle_layer_on_tokens
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


def mk_cfg(B, wl, T):
    return B.MoeConfig(T=T, H=wl.H, E=wl.E, k=wl.k, I=wl.I, n_shared=wl.n_shared,
                       n_group=wl.n_group, topk_group=wl.topk_group, group_topn=wl.group_topn,
                       norm_topk_prob=wl.norm_topk_prob,
                       routed_scaling_factor=wl.routed_scaling_factor)


def tokens_of(W, wl, N, T, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return [torch.randn((T, wl.H), generator=g, device="cuda").to(torch.bfloat16)
            for _ in range(N)]


def single_gpu_forward(B, cfg, inp, x):
    ws = B.alloc_workspace(cfg)
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    B.moe_forward(cfg, x, inp["w_router"], inp["bias"], inp["w13"], inp["w2"], inp["w13s"],
                  inp["w2s"], out, ws)
    B.moe_check_device_status(ws)
    return out, ws


def check_rank(B, cfg, inp, x, out, name, tokens=None):
    """The rank's output equals moe_forward's on the same tokens bit for bit:
    each routed row is one fp32 GEMM row times its weight, rounded once to
    bf16 on both paths (the expert side's k = 1 combine adds nothing to it),
    the shared expert's fp32 rows are the same whichever token tile computes
    them, and the final combine sums in the same slot order.  And it meets
    the bf16 bar against the oracle."""
    ref_gpu, ws = single_gpu_forward(B, cfg, inp, x)
    rel = (out.float() - ref_gpu.float()).norm() / ref_gpu.float().norm()
    same = (out == ref_gpu).float().mean().item()
    assert torch.equal(out, ref_gpu), "%s: %.4f%% bit-equal to moe_forward, rel-L2 %.2e" % (
        name, 100 * same, rel)
    idx = B.ws_view(ws, cfg, "topk_idx").cpu().numpy()
    w = B.ws_view(ws, cfg, "topk_w").cpu().numpy()
    toks = np.arange(cfg.T) if tokens is None else np.asarray(tokens)
    inp_r = dict(inp, x=x)
    ref = oracle_layer_on_tokens(cfg, inp_r, idx, w, toks)
    r, m = assert_close_bf16(out[torch.as_tensor(toks, device="cuda")].float().cpu().numpy(),
                             ref, name)
    return rel.item(), same, r, m


@pytest.mark.parametrize("N", [2, 4, 8])
def test_virtual_ranks_small(B, W, N):
    from sigmoid_top_routing_warp_b200 import ep
    wl = W.Workload("ep_small", T=96, H=512, E=256, k=8, I=128, n_shared=1, seed=13)
    inp = W.make_inputs(wl, device="cuda")
    xs = tokens_of(W, wl, N, wl.T, seed=40 + N)
    cfg = mk_cfg(B, wl, wl.T)
    outs = ep.ep_forward_virtual(cfg, xs, inp["w_router"], inp["bias"], inp["w13"], inp["w2"],
                                 inp["w13s"], inp["w2s"])
    torch.cuda.synchronize()
    for r in range(N):
        rel, same, orel, omx = check_rank(B, cfg, inp, xs[r], outs[r], "N=%d rank %d" % (N, r))
        print("N=%d rank %d: vs moe_forward rel-L2 %.1e (%.1f%% bit-equal), vs oracle rel-L2 "
              "%.2e max-abs/rms %.2e" % (N, r, rel, 100 * same, orel, omx))


def test_ep_pack_rows_weights_and_counts(B, W):
    """moe_ep_pack against the oracle's permutation: row r of the send buffer
    is token rows[r] of x, its weight and its expert's local index; the counts
    split the rows by owner."""
    wl = W.Workload("ep_pack", T=300, H=512, E=64, k=6, I=128, seed=5)
    inp = W.make_inputs(wl, device="cuda")
    cfg = mk_cfg(B, wl, wl.T)
    N = 4
    el = wl.E // N
    ws = B.alloc_workspace(cfg)
    T, k, E, H = wl.T, wl.k, wl.E, wl.H
    logits = torch.empty((T, E), device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), device="cuda")
    B.moe_route(cfg, inp["x"], inp["w_router"], inp["bias"], logits, idx, w, ws)
    offs = torch.empty((E + 1,), dtype=torch.int32, device="cuda")
    rows = torch.empty((T * k,), dtype=torch.int32, device="cuda")
    pos = torch.empty((T * k,), dtype=torch.int32, device="cuda")
    B.moe_permute(cfg, idx, offs, rows, pos, ws)
    xs = torch.empty((T * k, H), dtype=torch.bfloat16, device="cuda")
    wsend = torch.empty((T * k,), device="cuda")
    esend = torch.empty((T * k,), dtype=torch.int32, device="cuda")
    cnt = torch.empty((N,), dtype=torch.int32, device="cuda")
    B.moe_ep_pack(cfg, N, inp["x"], idx, w, offs, pos, xs, wsend, esend, cnt)
    torch.cuda.synchronize()
    i, wn = idx.cpu().numpy(), w.cpu().numpy()
    o_offs, o_rows, o_pos = O.permute(oracle_cfg(cfg), i)
    assert (cnt.cpu().numpy() == np.diff(o_offs[::el])).all()
    assert torch.equal(xs, inp["x"][torch.as_tensor(o_rows, device="cuda").long()])
    slot_of_row = np.empty(T * k, np.int64)
    slot_of_row[o_pos] = np.arange(T * k)
    assert (wsend.cpu().numpy().view(np.uint32) == wn.ravel()[slot_of_row].view(np.uint32)).all()
    assert (esend.cpu().numpy() == i.ravel()[slot_of_row] % el).all()


def test_shared_expert_alone_matches_the_layer(B, W):
    """moe_shared_expert gives the shared expert's fp32 output the whole layer
    computes beside the routed experts (both paths: single CTAs and pairs)."""
    for T in (200, 1500):
        wl = W.Workload("shared_only", T=T, H=640, E=32, k=4, I=384, n_shared=2, seed=17)
        inp = W.make_inputs(wl, device="cuda")
        cfg = mk_cfg(B, wl, T)
        _, ws = single_gpu_forward(B, cfg, inp, inp["x"])
        ref = B.ws_view(ws, cfg, "y_shared").float()
        ysh = torch.empty((T, wl.H), dtype=torch.float32, device="cuda")
        ws2 = B.alloc_workspace(cfg)
        B.moe_shared_expert(cfg, inp["x"], inp["w13s"], inp["w2s"], ysh, ws2)
        B.moe_check_device_status(ws2)
        rel = (ysh - ref).norm() / ref.norm()
        assert rel <= 1e-3, (T, rel.item())


def test_virtual_ranks_dots3_decode_shape(B, W):
    """The dots3 shape (H 5120, 256 experts top-8, I 1536, one shared) over 8
    virtual ranks of 32 experts each, 64 tokens per rank: every token of
    rank 0 against the oracle, every rank against moe_forward."""
    from sigmoid_top_routing_warp_b200 import ep
    wl = W.WORKLOADS["decode"]
    inp = W.make_inputs(wl, device="cuda")
    N = 8
    xs = [inp["x"]] + tokens_of(W, wl, N - 1, wl.T, seed=77)
    cfg = mk_cfg(B, wl, wl.T)
    outs = ep.ep_forward_virtual(cfg, xs, inp["w_router"], inp["bias"], inp["w13"], inp["w2"],
                                 inp["w13s"], inp["w2s"])
    torch.cuda.synchronize()
    for r in range(N):
        rel, same, orel, omx = check_rank(B, cfg, inp, xs[r], outs[r], "dots3 rank %d" % r,
                                          tokens=None if r == 0 else [0, wl.T - 1])
        print("dots3 N=8 rank %d: vs moe_forward rel-L2 %.1e (%.1f%% bit-equal), vs oracle "
              "rel-L2 %.2e max-abs/rms %.2e" % (r, rel, 100 * same, orel, omx))


@pytest.mark.parametrize("N", [2, 4, 8])
def test_peer_exchange_virtual_ranks_small(B, W, N):
    """The peer-memory form (moe_ep_expert_counts, moe_ep_plan,
    moe_ep_dispatch_peer, moe_ep_combine_peer) on N virtual ranks: every
    rank's output equals moe_forward's bit for bit."""
    from sigmoid_top_routing_warp_b200 import ep
    wl = W.Workload("ep_peer", T=96, H=512, E=256, k=8, I=128, n_shared=1, seed=19)
    inp = W.make_inputs(wl, device="cuda")
    xs = tokens_of(W, wl, N, wl.T, seed=60 + N)
    cfg = mk_cfg(B, wl, wl.T)
    outs = ep.ep_forward_peer_virtual(cfg, xs, inp["w_router"], inp["bias"], inp["w13"],
                                      inp["w2"], inp["w13s"], inp["w2s"])
    torch.cuda.synchronize()
    for r in range(N):
        check_rank(B, cfg, inp, xs[r], outs[r], "peer N=%d rank %d" % (N, r),
                   tokens=[0, wl.T // 2, wl.T - 1])


def test_peer_exchange_dots3_decode_shape(B, W):
    """The dots3 decode shape over 8 virtual ranks of 32 experts with the
    peer-memory exchange: bit-identical to moe_forward on every rank."""
    from sigmoid_top_routing_warp_b200 import ep
    wl = W.WORKLOADS["decode"]
    inp = W.make_inputs(wl, device="cuda")
    N = 8
    xs = [inp["x"]] + tokens_of(W, wl, N - 1, wl.T, seed=91)
    cfg = mk_cfg(B, wl, wl.T)
    outs = ep.ep_forward_peer_virtual(cfg, xs, inp["w_router"], inp["bias"], inp["w13"],
                                      inp["w2"], inp["w13s"], inp["w2s"])
    torch.cuda.synchronize()
    for r in range(N):
        check_rank(B, cfg, inp, xs[r], outs[r], "peer dots3 rank %d" % r,
                   tokens=None if r == 0 else [0, wl.T - 1])


def test_peer_plan_flags_a_receive_buffer_too_small(B, W):
    """Rows beyond a rank's receive capacity are dropped and flagged in the
    status word: moe_check_device_status reports MOE_ERR_WORKSPACE."""
    wl = W.Workload("ep_cap", T=64, H=512, E=64, k=4, I=128, seed=23)
    inp = W.make_inputs(wl, device="cuda")
    cfg = mk_cfg(B, wl, wl.T)
    ws = B.alloc_workspace(cfg)
    N, el = 2, 32
    counts_all = torch.full((N, wl.E), 5, dtype=torch.int32, device="cuda")  # 320 rows per rank
    eb = torch.empty((wl.E,), dtype=torch.int32, device="cuda")
    sb = torch.empty_like(eb)
    ro = torch.empty((el + 1,), dtype=torch.int32, device="cuda")
    ident = torch.empty((100,), dtype=torch.int32, device="cuda")
    B.moe_ep_plan(cfg, N, 1, counts_all, eb, sb, ro, ident, 100, ws)
    with pytest.raises(B.MoeError) as ei:
        B.moe_check_device_status(ws)
    assert ei.value.status == B.MOE_ERR_WORKSPACE
    # the plan itself: expert-major layout, sources in rank order
    assert (eb.cpu().numpy() == np.tile(np.arange(el) * 10, N)).all()
    assert (sb.cpu().numpy() == 5).all()
    assert (ro.cpu().numpy() == np.arange(el + 1) * 10).all()
    assert (ident.cpu().numpy() == np.arange(100)).all()


@pytest.mark.parametrize("form", ["all_to_all", "peer"])
def test_every_choice_on_one_rank(B, W, form):
    """A bias that puts every token's choice among rank 0's experts: the other
    ranks own experts nobody chose and receive no rows (empty exchanges and
    empty expert segments on three of four ranks); every rank's output still
    equals moe_forward's bit for bit."""
    from sigmoid_top_routing_warp_b200 import ep
    wl = W.Workload("ep_skew", T=80, H=512, E=128, k=4, I=128, n_shared=1, seed=29)
    inp = W.make_inputs(wl, device="cuda")
    N = 4
    bias = torch.full((wl.E,), -20.0, device="cuda")
    bias[: wl.E // N] = 20.0  # rank 0's 32 experts win every choice
    inp = dict(inp, bias=bias)
    xs = tokens_of(W, wl, N, wl.T, seed=77)
    cfg = mk_cfg(B, wl, wl.T)
    run = ep.ep_forward_peer_virtual if form == "peer" else ep.ep_forward_virtual
    outs = run(cfg, xs, inp["w_router"], inp["bias"], inp["w13"], inp["w2"], inp["w13s"], inp["w2s"])
    torch.cuda.synchronize()
    for r in range(N):
        check_rank(B, cfg, inp, xs[r], outs[r], "%s skewed rank %d" % (form, r),
                   tokens=[0, wl.T // 2, wl.T - 1])

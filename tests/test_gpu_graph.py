"""CUDA graph capture of the C-ABI calls: a captured moe_forward /
moe_forward_block / dsa_indexer replays to the same bits as the eager call
(the library enqueues only kernels, copies none and allocates nothing, so a
stream capture records the whole layer)."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from sigmoid_top_routing_warp_b200 import binding
    return binding


@pytest.fixture(scope="module")
def W():
    from sigmoid_top_routing_warp_b200 import workloads
    return workloads


def mk_cfg(B, wl):
    return B.MoeConfig(T=wl.T, H=wl.H, E=wl.E, k=wl.k, I=wl.I, n_shared=wl.n_shared,
                       n_group=wl.n_group, topk_group=wl.topk_group,
                       dtype=B.MOE_DTYPE_FP8_E4M3_BLOCK128 if wl.dtype == "fp8" else B.MOE_DTYPE_BF16)


def scales(inp):
    return {k: inp.get(k) for k in ("w13_scale", "w2_scale", "w13s_scale", "w2s_scale")}


@pytest.mark.parametrize("name,T", [("decode", None), ("prefill", 1024), ("fp8_256", None)])
def test_forward_graph_replay_is_bit_identical(B, W, name, T):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, device="cuda", T=T)
    if T is not None:
        from dataclasses import replace
        wl = replace(wl, T=T)
    cfg = mk_cfg(B, wl)
    ws = B.alloc_workspace(cfg)
    out_eager = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    out_graph = torch.empty_like(out_eager)
    B.moe_forward(cfg, inp["x"], inp["w_router"], inp["bias"], inp["w13"], inp["w2"], inp["w13s"],
                  inp["w2s"], out_eager, ws, **scales(inp))
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            B.moe_forward(cfg, inp["x"], inp["w_router"], inp["bias"], inp["w13"], inp["w2"],
                          inp["w13s"], inp["w2s"], out_graph, ws, stream=s, **scales(inp))
    for _ in range(3):
        out_graph.zero_()
        g.replay()
    torch.cuda.synchronize()
    B.moe_check_device_status(ws)
    assert torch.equal(out_graph, out_eager)
    del g


def test_block_and_indexer_graph_replay(B, W):
    wl = W.WORKLOADS["tiny"]
    inp = W.make_inputs(wl, device="cuda")
    gamma = W.make_norm_weight(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    ws = B.alloc_workspace(cfg)
    ref = torch.empty_like(inp["x"])
    got = torch.empty_like(inp["x"])
    B.moe_forward_block(cfg, inp["x"], gamma, W.RMS_NORM_EPS, inp["w_router"], inp["bias"],
                        inp["w13"], inp["w2"], inp["w13s"], inp["w2s"], ref, ws)
    dwl = W.DSA_WORKLOADS["dsa_tiny"]
    din = W.make_dsa_inputs(dwl, device="cuda")
    dcfg = B.DsaConfig(Sq=dwl.Sq, Sk=dwl.Sk, n_heads=dwl.n_heads, topk=dwl.topk, causal=dwl.causal)
    dws = B.dsa_alloc_workspace(dcfg)
    idx_ref = torch.empty((dwl.Sq, dwl.topk), dtype=torch.int32, device="cuda")
    idx_got = torch.empty_like(idx_ref)
    B.dsa_indexer(dcfg, din["q"], din["k"], din["w"], idx_ref, dws)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            B.moe_forward_block(cfg, inp["x"], gamma, W.RMS_NORM_EPS, inp["w_router"], inp["bias"],
                                inp["w13"], inp["w2"], inp["w13s"], inp["w2s"], got, ws, stream=s)
            B.dsa_indexer(dcfg, din["q"], din["k"], din["w"], idx_got, dws, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(got, ref) and torch.equal(idx_got, idx_ref)
    del g

"""GPU parity of the FP8 layer (e4m3 weights with 128x128 block scales,
activations quantised per token and 128 columns) against the CPU oracle in
fp8 mode.  Step a0 (the quantisation itself) must match bit for bit; routing
stays bf16 and bit-exact; the layer output must reach relative L2 <= 3e-2."""
import numpy as np
import pytest
import torch

from helpers import (assert_close_fp8, check_routing_fn, cover_tokens,
                     oracle_layer_on_tokens)
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


def mk_cfg(B, wl):
    return B.MoeConfig(T=wl.T, H=wl.H, E=wl.E, k=wl.k, I=wl.I, n_shared=wl.n_shared,
                       n_group=wl.n_group, topk_group=wl.topk_group, group_topn=wl.group_topn,
                       norm_topk_prob=wl.norm_topk_prob,
                       routed_scaling_factor=wl.routed_scaling_factor,
                       dtype=B.MOE_DTYPE_FP8_E4M3_BLOCK128)


def run_forward(B, cfg, inp):
    ws = B.alloc_workspace(cfg)
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    B.moe_forward(cfg, inp["x"], inp["w_router"], inp["bias"], inp["w13"], inp["w2"],
                  inp.get("w13s"), inp.get("w2s"), out, ws, w13_scale=inp["w13_scale"],
                  w2_scale=inp["w2_scale"], w13s_scale=inp.get("w13s_scale"),
                  w2s_scale=inp.get("w2s_scale"))
    B.moe_check_device_status(ws)
    return out, ws


def test_activation_quantisation_bit_exact(B):
    g = torch.Generator(device="cuda").manual_seed(5)
    rows, cols = 77, 1280
    x = (torch.randn((rows, cols), generator=g, device="cuda") * 3).to(torch.bfloat16)
    x[3, 128:256] = 0                      # all-zero block -> scale 1, codes 0
    x[5, :128] *= 1000                     # large values
    x[6, 256:384] *= 1e-3                  # small values
    x[7, 0] = -0.0
    q = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    s = torch.empty((rows, cols // 128), dtype=torch.float32, device="cuda")
    B.moe_quantize_act(x, q, s)
    torch.cuda.synchronize()
    oq, os_ = O.quant_act_e4m3(x.float().cpu().numpy())
    assert (s.cpu().numpy().view(np.uint32) == os_.view(np.uint32)).all()
    assert (q.cpu().numpy() == oq).all()
    assert (s[3, 1] == 1).item() and (q[3, 128:256] == 0).all()


SMALL = [
    # name, T, H, E, k, I, n_shared  (weight-major token tiles of 16, 32 and 64,
    # ragged: I or H not a multiple of 512 keeps these off the token-major kernel)
    ("fp8_small", 96, 512, 32, 4, 256, 1),
    ("fp8_tiles64", 700, 768, 32, 6, 384, 2),
    ("fp8_tiles32", 200, 512, 32, 6, 256, 1),
    ("fp8_one_token", 1, 512, 32, 8, 128, 1),
    # token-major kernel (H and I multiples of 512): ragged 128-row tiles,
    # experts over two tiles, one K group in the down GEMM, 8 rows per expert,
    # a single token
    ("fp8_tokmajor", 1200, 1024, 32, 4, 512, 1),
    ("fp8_tokmajor_sparse", 64, 1024, 32, 4, 512, 1),
    ("fp8_tokmajor_one_token", 1, 512, 32, 8, 512, 1),
    ("fp8_tokmajor_s2", 700, 1536, 32, 8, 512, 2),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_fp8_layer_small(B, W, case):
    name, T, H, E, k, I, S = case
    wl = W.Workload(name, T=T, H=H, E=E, k=k, I=I, n_shared=S, dtype="fp8",
                    seed=sum(name.encode()) % 1000)
    inp = W.make_inputs(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    out, ws = run_forward(B, cfg, inp)
    L, idx, w, ties = check_routing_fn(B, cfg, ws, inp)
    ref = oracle_layer_on_tokens(cfg, inp, idx, w, np.arange(T))
    rel = assert_close_fp8(out.float().cpu().numpy(), ref, name)
    print("%s: rel-L2 %.2e, near-ties %d" % (name, rel, ties))


@pytest.mark.parametrize("name", ["fp8_256", "fp8_4096"])
def test_fp8_full_size(B, W, name):
    """Every token at T = 256; at T = 4096 a token of every expert and the last
    row of every 128-row token tile (the token-major GEMMs' tiles)."""
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    out, ws = run_forward(B, cfg, inp)
    L, idx, w, ties = check_routing_fn(B, cfg, ws, inp)
    if cfg.T <= 256:
        toks = np.arange(cfg.T)
    else:
        offs = B.ws_view(ws, cfg, "offsets").cpu().numpy()
        toks = cover_tokens(offs, B.ws_view(ws, cfg, "rows").cpu().numpy(), 128)
        assert np.isin(np.arange(cfg.E)[np.diff(offs) > 0], np.unique(idx[toks])).all()
    ref = oracle_layer_on_tokens(cfg, inp, idx, w, toks)
    got = out[torch.as_tensor(toks, device="cuda")].float().cpu().numpy()
    rel = assert_close_fp8(got, ref, name)
    assert ties <= cfg.T // 20 + 2, "near-ties %d of %d tokens" % (ties, cfg.T)
    print("%s: %d tokens compared, rel-L2 %.2e, near-ties %d/%d" % (name, toks.size, rel, ties,
                                                                     cfg.T))


@pytest.mark.parametrize("case", [c for c in SMALL if c[0] in ("fp8_tokmajor", "fp8_tokmajor_sparse")],
                         ids=lambda c: c[0])
def test_token_major_claim_counters_reset_and_repeat(B, W, case):
    """The token-major fp8 GEMMs claim tiles from counters in the workspace
    status block (words 24..29): a call leaves them at zero, and repeated calls
    on one workspace give the same output bit for bit."""
    name, T, H, E, k, I, S = case
    wl = W.Workload(name, T=T, H=H, E=E, k=k, I=I, n_shared=S, dtype="fp8")
    inp = W.make_inputs(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    out1, ws = run_forward(B, cfg, inp)
    assert (ws[:256].view(torch.int32).cpu().numpy()[16:30] == 0).all()
    out2 = torch.empty_like(out1)
    for _ in range(3):
        B.moe_forward(cfg, inp["x"], inp["w_router"], inp["bias"], inp["w13"], inp["w2"],
                      inp.get("w13s"), inp.get("w2s"), out2, ws, w13_scale=inp["w13_scale"],
                      w2_scale=inp["w2_scale"], w13s_scale=inp.get("w13s_scale"),
                      w2s_scale=inp.get("w2s_scale"))
    B.moe_check_device_status(ws)
    assert torch.equal(out1, out2)
    assert (ws[:256].view(torch.int32).cpu().numpy()[16:30] == 0).all()

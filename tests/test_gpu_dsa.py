"""DSA indexer on the GPU against the oracle (include/dsa.h).

- Selection: bit-exact.  The top-k kernel and the oracle's selection are
  given the same fp32 scores and must return the same indices (score
  descending, equal scores by lower key, -1 padding).
- Scores: fp32 accumulation of exact bf16 products against the oracle's fp64
  sum; bound 1e-5 of the row's largest |score| plus 1e-5 of the entry's own
  magnitude bound (sum_h |w| * |q.k|); masked entries exactly -inf.
- End to end: the chosen set against the oracle's fp64 ranking, up to keys
  whose fp64 score lies within that bound of the k-th score (near-ties may
  fall either way).
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.helpers import u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from sigmoid_top_routing_warp_b200 import binding
    return binding


@pytest.fixture(scope="module")
def W():
    from sigmoid_top_routing_warp_b200 import workloads
    return workloads


def cfg_of(B, wl, **kw):
    base = dict(Sq=wl.Sq, Sk=wl.Sk, n_heads=wl.n_heads, topk=wl.topk, causal=wl.causal,
                q_offset=wl.q_offset)
    base.update(kw)
    return B.DsaConfig(**base)


@pytest.mark.parametrize("Sq,Sk,topk", [(64, 100, 7), (33, 4096, 2048), (17, 40000, 2048),
                                        (8, 3000, 1), (5, 2047, 2048)])
def test_topk_bit_exact(B, Sq, Sk, topk):
    g = torch.Generator(device="cuda").manual_seed(Sk + topk)
    sc = torch.randint(-50, 50, (Sq, Sk), generator=g, device="cuda").float() * 0.25  # many ties
    sc[0, : Sk // 2] = float("-inf")
    sc[1, 3] = float("nan")
    if Sq > 2:
        sc[2] = torch.randn(Sk, generator=g, device="cuda")
    idx = torch.empty((Sq, topk), dtype=torch.int32, device="cuda")
    B.dsa_index_topk(B.DsaConfig(Sq=Sq, Sk=Sk, n_heads=1, topk=topk), sc, idx)
    torch.cuda.synchronize()
    ref = O.dsa_topk(sc.cpu().numpy(), topk)
    assert np.array_equal(idx.cpu().numpy(), ref)
    # index-ordered output: the same set, ascending, -1 padding last
    B.dsa_index_topk(B.DsaConfig(Sq=Sq, Sk=Sk, n_heads=1, topk=topk, sorted=False), sc, idx)
    torch.cuda.synchronize()
    ref_set = np.sort(np.where(ref < 0, np.iinfo(np.int32).max, ref), axis=1)
    ref_set = np.where(ref_set == np.iinfo(np.int32).max, -1, ref_set)
    assert np.array_equal(idx.cpu().numpy(), ref_set)


@pytest.mark.parametrize("Sk,topk,cached", [(20000, 2048, True), (36000, 1000, False)])
def test_topk_one_top_digit(B, Sk, topk, cached):
    """Scores in [1, 2) share their top radix digit, so the candidate buffer
    overflows and the later digits scan the whole row; distinct scores take
    the unordered gather before the sort; a few duplicated values sit at
    random places (ties at the threshold go by lower index)."""
    Sq = 6
    g = torch.Generator(device="cuda").manual_seed(Sk)
    sc = 1.0 + torch.rand((Sq, Sk), generator=g, device="cuda")
    sc[1] = sc[1].sort(descending=True).values  # the k-th largest inside a sorted run
    sc[2, ::7] = sc[2, 5]                         # one value repeated many times
    sc[3, : Sk - topk // 2] = float("-inf")       # fewer valid keys than k
    assert (Sk <= 32768) == cached
    idx = torch.empty((Sq, topk), dtype=torch.int32, device="cuda")
    ref = O.dsa_topk(sc.cpu().numpy(), topk)
    for srt in (True, False):
        B.dsa_index_topk(B.DsaConfig(Sq=Sq, Sk=Sk, n_heads=1, topk=topk, sorted=srt), sc, idx)
        torch.cuda.synchronize()
        want = ref if srt else np.sort(np.where(ref < 0, Sk, ref), axis=1)
        want = np.where(want == Sk, -1, want)
        assert np.array_equal(idx.cpu().numpy(), want), srt


def test_indexer_causal_small(B, W):
    """Causal rows with a query offset: each row reads only its unmasked keys
    (the rest are the score kernel's -inf); selection bit-exact on the GPU's
    scores, both output orders."""
    wl = W.DsaWorkload("t", Sq=300, Sk=2500, n_heads=4, topk=256, causal=True, q_offset=2150,
                       seed=11)
    inp = W.make_dsa_inputs(wl, device="cuda")
    for srt in (True, False):
        cfg = cfg_of(B, wl, sorted=srt)
        ws = B.dsa_alloc_workspace(cfg)
        idx = torch.empty((wl.Sq, wl.topk), dtype=torch.int32, device="cuda")
        B.dsa_indexer(cfg, inp["q"], inp["k"], inp["w"], idx, ws)
        B.moe_check_device_status(ws)
        gsc = B.dsa_scores_view(ws, cfg).cpu().numpy()
        ref = O.dsa_topk(gsc, wl.topk)
        if not srt:
            ref = np.sort(ref, axis=1)
        assert np.array_equal(idx.cpu().numpy(), ref), srt


def score_bound(q, k, w, rows, causal, q_offset):
    """|error| bound per entry: 1e-5 * (row max |score| + sum_h |w| |q.k|)."""
    qf = q.float()[rows].double()
    kf = k.float().double()
    dots = torch.einsum("thd,shd->tsh", qf, kf)
    mag = torch.einsum("tsh,th->ts", dots.abs(), w.float()[rows].double().abs())
    return mag.cpu().numpy()


@pytest.mark.parametrize("Sq,Sk,nh,causal,q_offset", [(200, 600, 8, False, 0),
                                                      (130, 300, 64, True, 0),
                                                      (77, 513, 4, True, 400),
                                                      (256, 1024, 2, True, 768)])
def test_scores_against_oracle(B, W, Sq, Sk, nh, causal, q_offset):
    wl = W.DsaWorkload("t", Sq=Sq, Sk=Sk, n_heads=nh, topk=16, causal=causal, q_offset=q_offset,
                       seed=Sq + Sk)
    inp = W.make_dsa_inputs(wl, device="cuda")
    cfg = cfg_of(B, wl)
    ws = B.dsa_alloc_workspace(cfg)
    scores = torch.empty((Sq, Sk), dtype=torch.float32, device="cuda")
    B.dsa_index_scores(cfg, inp["q"], inp["k"], inp["w"], scores, ws)
    B.moe_check_device_status(ws)
    got = scores.cpu().numpy().astype(np.float64)
    ref = O.dsa_scores(u16(inp["q"]), u16(inp["k"]), u16(inp["w"]), causal, q_offset)
    masked = np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), masked)
    mag = score_bound(inp["q"], inp["k"], inp["w"], np.arange(Sq), causal, q_offset)
    rowmax = np.where(masked, 0.0, np.abs(ref)).max(axis=1, keepdims=True)
    tol = 1e-5 * (rowmax + mag)
    err = np.abs(np.where(masked, 0.0, got) - np.where(masked, 0.0, ref))
    assert (err <= tol).all(), "max err %.3e (tol %.3e)" % (err.max(), tol[err > tol].min())


def check_selection(idx_row, ref_row, tol_row, topk):
    """idx_row: GPU indices; ref_row: fp64 scores; every key clearly above the
    k-th score is chosen, none clearly below it, no key twice."""
    valid = np.where(np.isfinite(ref_row))[0]
    want = min(topk, valid.size)
    chosen = idx_row[:want]
    assert (idx_row[want:] == -1).all()
    assert len(set(chosen.tolist())) == want and np.isfinite(ref_row[chosen]).all()
    if want < valid.size:
        kth = np.sort(ref_row[valid])[::-1][want - 1]
        clearly_in = valid[ref_row[valid] > kth + tol_row[valid]]
        clearly_out = valid[ref_row[valid] < kth - tol_row[valid]]
        cs = set(chosen.tolist())
        assert all(s in cs for s in clearly_in.tolist())
        assert not any(s in cs for s in clearly_out.tolist())


def test_indexer_small_end_to_end(B, W):
    wl = W.DSA_WORKLOADS["dsa_tiny"]
    inp = W.make_dsa_inputs(wl, device="cuda")
    cfg = cfg_of(B, wl)
    ws = B.dsa_alloc_workspace(cfg)
    idx = torch.empty((wl.Sq, wl.topk), dtype=torch.int32, device="cuda")
    B.dsa_indexer(cfg, inp["q"], inp["k"], inp["w"], idx, ws)
    B.moe_check_device_status(ws)
    got = idx.cpu().numpy()
    # bit-exact against the oracle's selection on the GPU's own scores
    gsc = B.dsa_scores_view(ws, cfg).cpu().numpy()
    assert np.array_equal(got, O.dsa_topk(gsc, wl.topk))
    ref = O.dsa_scores(u16(inp["q"]), u16(inp["k"]), u16(inp["w"]), wl.causal, wl.q_offset)
    mag = score_bound(inp["q"], inp["k"], inp["w"], np.arange(wl.Sq), wl.causal, wl.q_offset)
    for t in range(wl.Sq):
        check_selection(got[t], ref[t], 2e-5 * (np.abs(ref[t][np.isfinite(ref[t])]).max() + mag[t]),
                        wl.topk)


@pytest.mark.parametrize("name,sample", [("dsa_prefill", 4), ("dsa_long", 4)])
def test_indexer_full_size_sampled(B, W, name, sample):
    wl = W.DSA_WORKLOADS[name]
    inp = W.make_dsa_inputs(wl, device="cuda")
    cfg = cfg_of(B, wl)
    ws = B.dsa_alloc_workspace(cfg)
    idx = torch.empty((wl.Sq, wl.topk), dtype=torch.int32, device="cuda")
    B.dsa_indexer(cfg, inp["q"], inp["k"], inp["w"], idx, ws)
    B.moe_check_device_status(ws)
    rows = np.unique(np.concatenate([np.random.default_rng(2).choice(wl.Sq, sample, replace=False),
                                     [0, wl.Sq - 1]]))
    gsc = B.dsa_scores_view(ws, cfg)[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    got = idx[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    assert np.array_equal(got, O.dsa_topk(gsc, wl.topk))
    q_rows = inp["q"][torch.as_tensor(rows, device="cuda")]
    w_rows = inp["w"][torch.as_tensor(rows, device="cuda")]
    for n, t in enumerate(rows):
        # the oracle row of query t: its absolute position is q_offset + t
        ref = O.dsa_scores(u16(q_rows[n:n + 1]), u16(inp["k"]), u16(w_rows[n:n + 1]), wl.causal,
                           wl.q_offset + int(t))[0]
        mag = score_bound(q_rows[n:n + 1], inp["k"], w_rows[n:n + 1], [0], wl.causal, 0)[0]
        fin = np.isfinite(ref)
        assert np.array_equal(np.isneginf(gsc[n]), ~fin)
        tol = 1e-5 * (np.abs(ref[fin]).max() + mag)
        assert (np.abs(gsc[n][fin] - ref[fin]) <= tol[fin]).all()
        check_selection(got[n], ref, 2 * tol, wl.topk)


def test_score_claim_counters_reset_and_repeat(B, W):
    """The score kernel claims tiles from counters in the workspace status
    block (words 16..17): a call leaves them at zero, and repeated calls on one
    workspace give the same scores and indices bit for bit."""
    wl = W.DsaWorkload("t", Sq=700, Sk=1900, n_heads=4, topk=128, causal=True, q_offset=300, seed=3)
    inp = W.make_dsa_inputs(wl, device="cuda")
    cfg = cfg_of(B, wl)
    ws = B.dsa_alloc_workspace(cfg)
    idx1 = torch.empty((wl.Sq, wl.topk), dtype=torch.int32, device="cuda")
    B.dsa_indexer(cfg, inp["q"], inp["k"], inp["w"], idx1, ws)
    B.moe_check_device_status(ws)
    sc1 = B.dsa_scores_view(ws, cfg).clone()
    assert (ws[:256].view(torch.int32).cpu().numpy()[16:18] == 0).all()
    idx2 = torch.empty_like(idx1)
    for _ in range(3):
        B.dsa_indexer(cfg, inp["q"], inp["k"], inp["w"], idx2, ws)
    B.moe_check_device_status(ws)
    assert torch.equal(sc1.view(torch.int32), B.dsa_scores_view(ws, cfg).view(torch.int32))
    assert torch.equal(idx1, idx2)
    assert (ws[:256].view(torch.int32).cpu().numpy()[16:18] == 0).all()

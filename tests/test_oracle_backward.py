"""Pins of the fp64 backward-pass reference (oracle/backward.py).

Its forward pass is pinned to the C oracle's layer and routing weights; its
gradients are pinned by central finite differences of that forward pass, by
closed forms (k = 1 with renormalisation has no router gradient) and by
invariants.  No GPU is used.
"""
import numpy as np
import pytest

from oracle import backward as BW
from oracle import oracle as O


def bf16_round(a):
    """fp64 -> the nearest bf16 value (as fp64) and its bit pattern."""
    bits = O.f64_to_bf16(np.ascontiguousarray(a, np.float64))
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64), bits


def choose(s, b, k):
    """top-k of s + b, larger first, lower index on ties (the layer's rule)."""
    c = s + b
    return np.argsort(-c, axis=1, kind="stable")[:, :k]


def small_case(seed, T=5, H=16, E=6, k=2, I=8, Is=8, scale=0.3):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H))
    wg = rng.standard_normal((E, H)) * scale
    w13 = rng.standard_normal((E, 2 * I, H)) * scale
    w2 = rng.standard_normal((E, H, I)) * scale
    w13s = rng.standard_normal((2 * Is, H)) * scale if Is else None
    w2s = rng.standard_normal((H, Is)) * scale if Is else None
    b = rng.uniform(-0.1, 0.1, E)
    s = 1.0 / (1.0 + np.exp(-(x @ wg.T)))
    idx = choose(s, b, k)
    return dict(x=x, wg=wg, w13=w13, w2=w2, w13s=w13s, w2s=w2s, b=b, idx=idx, rng=rng)


# ------------------------------------------------------------------ forward pins

def test_forward_matches_the_c_oracle_layer_and_routing():
    rng = np.random.default_rng(3)
    T, H, E, k, I, Is = 6, 128, 8, 3, 128, 128
    x, xb = bf16_round(rng.standard_normal((T, H)))
    wg, wgb = bf16_round(rng.standard_normal((E, H)) * 0.05)
    w13, w13b = bf16_round(rng.standard_normal((E, 2 * I, H)) * 0.05)
    w2, w2b = bf16_round(rng.standard_normal((E, H, I)) * 0.05)
    w13s, w13sb = bf16_round(rng.standard_normal((2 * Is, H)) * 0.05)
    w2s, w2sb = bf16_round(rng.standard_normal((H, Is)) * 0.05)
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    cfg = O.Config(T=T, H=H, E=E, k=k, I=I, n_shared=1)
    logits = O.router_logits(cfg, xb, wgb).astype(np.float32)
    idx, w32, _ = O.route(cfg, logits, bias)
    out, cache = BW.forward(x, wg, w13, w2, w13s, w2s, idx)
    # routing weights: fp64 here, fp32 (the GPU's arithmetic) in the C oracle
    assert np.allclose(cache["w"], w32, rtol=2e-6, atol=0)
    ref = O.layer(cfg, xb, idx, cache["w"].astype(np.float32), w13b, w2b, w13sb, w2sb)
    # the only difference is the routing weights' fp32 rounding
    assert np.abs(out - ref).max() <= 1e-6 * np.abs(ref).max()


# ------------------------------------------------------------------ gradient pins

@pytest.mark.parametrize("norm,rsf,shared", [(True, 1.0, True), (False, 2.5, True),
                                             (True, 0.5, False)])
def test_gradients_against_central_differences(norm, rsf, shared):
    c = small_case(11, Is=8 if shared else 0)
    rng = c["rng"]
    T, H = c["x"].shape
    dout = rng.standard_normal((T, H))
    args = dict(x=c["x"], wg=c["wg"], w13=c["w13"], w2=c["w2"], w13s=c["w13s"], w2s=c["w2s"])
    g = BW.backward(**args, idx=c["idx"], dout=dout, norm_topk_prob=norm, rsf=rsf)
    grads = dict(x=g["dx"], wg=g["dwg"], w13=g["dw13"], w2=g["dw2"], w13s=g["dw13s"],
                 w2s=g["dw2s"])

    def loss(a):
        out, _ = BW.forward(**a, idx=c["idx"], norm_topk_prob=norm, rsf=rsf)
        return float((out * dout).sum())

    eps = 1e-6
    for name, grad in grads.items():
        if args[name] is None:
            assert grad is None
            continue
        flat = args[name].reshape(-1)
        for p in rng.choice(flat.size, size=min(12, flat.size), replace=False):
            saved = flat[p]
            flat[p] = saved + eps
            lp = loss(args)
            flat[p] = saved - eps
            lm = loss(args)
            flat[p] = saved
            fd = (lp - lm) / (2 * eps)
            an = grad.reshape(-1)[p]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, p, fd, an)
    # the choice did not move under the perturbations (the gradients hold for it)
    s = 1.0 / (1.0 + np.exp(-(c["x"] @ c["wg"].T)))
    assert (choose(s, c["b"], c["idx"].shape[1]) == c["idx"]).all()


def test_one_renormalised_expert_has_no_router_gradient():
    """k = 1 with renormalisation: w = rsf whatever the score, so the
    router's logits and weight get no gradient (closed form)."""
    c = small_case(5, k=1)
    dout = c["rng"].standard_normal(c["x"].shape)
    g = BW.backward(c["x"], c["wg"], c["w13"], c["w2"], c["w13s"], c["w2s"], c["idx"], dout)
    assert np.abs(g["dlogits"]).max() < 1e-12
    assert np.abs(g["dwg"]).max() < 1e-12


def test_renormalised_weights_are_scale_free():
    """Scaling every chosen score by the same factor leaves the weights
    unchanged, so the score gradient is orthogonal to the scores."""
    c = small_case(7, k=3)
    dout = c["rng"].standard_normal(c["x"].shape)
    g = BW.backward(c["x"], c["wg"], c["w13"], c["w2"], c["w13s"], c["w2s"], c["idx"], dout)
    s = 1.0 / (1.0 + np.exp(-(c["x"] @ c["wg"].T)))
    ds = g["dlogits"] / (s * (1.0 - s))
    ssel = np.take_along_axis(s, c["idx"], 1)
    dssel = np.take_along_axis(ds, c["idx"], 1)
    assert np.abs((dssel * ssel).sum(1)).max() < 1e-12
    # off the chosen experts the logits get nothing
    mask = np.ones_like(s, dtype=bool)
    np.put_along_axis(mask, c["idx"], False, 1)
    assert (g["dlogits"][mask] == 0).all()


def test_backward_is_linear_in_the_upstream_gradient():
    c = small_case(9)
    rng = c["rng"]
    d1, d2 = rng.standard_normal(c["x"].shape), rng.standard_normal(c["x"].shape)
    args = (c["x"], c["wg"], c["w13"], c["w2"], c["w13s"], c["w2s"], c["idx"])
    g1, g2, g12 = (BW.backward(*args, d) for d in (d1, d2, d1 + 2.0 * d2))
    for key in ("dx", "dwg", "dw13", "dw2", "dw13s", "dw2s", "dw"):
        assert np.allclose(g12[key], g1[key] + 2.0 * g2[key], rtol=1e-12, atol=1e-12)


def test_expert_grads_equal_the_full_backward_per_expert():
    """expert_grads (one expert's weight gradients from its rows alone) equals
    backward()'s dw13[e] and dw2[e] for every expert, with the rows' routing
    weights, and the shared expert's dw13s / dw2s with weight 1 over every
    token; a dropped routing weight or a swapped gate/up half fails it."""
    c = small_case(11, T=9, H=16, E=5, k=2, I=6, Is=6)
    dout = c["rng"].standard_normal((9, 16))
    ref = BW.backward(c["x"], c["wg"], c["w13"], c["w2"], c["w13s"], c["w2s"], c["idx"], dout)
    _, cache = BW.forward(c["x"], c["wg"], c["w13"], c["w2"], c["w13s"], c["w2s"], c["idx"])
    for e in range(5):
        t, j = np.nonzero(c["idx"] == e)
        dw13, dw2 = BW.expert_grads(c["x"][t], dout[t], cache["w"][t, j], c["w13"][e], c["w2"][e])
        assert np.allclose(dw13, ref["dw13"][e], rtol=1e-12, atol=1e-12)
        assert np.allclose(dw2, ref["dw2"][e], rtol=1e-12, atol=1e-12)
        if t.size:
            bad13, bad2 = BW.expert_grads(c["x"][t], dout[t], np.ones(t.size), c["w13"][e],
                                          c["w2"][e])
            assert not np.allclose(bad2, ref["dw2"][e])
            swapped = np.concatenate([c["w13"][e][6:], c["w13"][e][:6]])
            bad13, _ = BW.expert_grads(c["x"][t], dout[t], cache["w"][t, j], swapped, c["w2"][e])
            assert not np.allclose(bad13, ref["dw13"][e])
    dw13s, dw2s = BW.expert_grads(c["x"], dout, np.ones(9), c["w13s"], c["w2s"])
    assert np.allclose(dw13s, ref["dw13s"], rtol=1e-12, atol=1e-12)
    assert np.allclose(dw2s, ref["dw2s"], rtol=1e-12, atol=1e-12)

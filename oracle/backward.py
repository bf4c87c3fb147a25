"""fp64 reference of the MoE layer's backward pass (the training side of the
layer: gradients of a loss through the routed SwiGLU experts, the shared
expert, the renormalised routing weights and the sigmoid router).

TEST INFRASTRUCTURE ONLY, like ``oracle.py``: imported by the test suite,
never by the product library (whose moe_backward it checks).

What it follows.  The forward pass is the one the pages describe ("Xiaohongshu
dots3 note Open Source Deep Dive", §3.1 Expert Routing Mechanism: gate ->
scores -> top-k -> renormalise -> shared + weighted routed sum; "dots3-note
架构深度解析" (mlqm.cn), 稀疏激活: sigmoid scores, noaux_tc, norm_topk_prob;
SwiGLU experts per §8.2 gmm1 -> swiglu -> gmm2).  The pages give no backward
pass; its definition is the chain rule through that forward pass, written
out step by step below:

  L = x W_g^T,  s = sigmoid(L),  c = s + b  (b steers the choice only)
  idx = top-k of c (piecewise constant: no gradient through the choice)
  S = sum_j s[idx_j],  w_j = rsf * s[idx_j] / S   (norm_topk_prob; else rsf * s[idx_j])
  g_j = x Wgate_e^T,  u_j = x Wup_e^T,  a_j = SiLU(g_j) * u_j,  y_j = a_j W2_e^T
  out = sum_j w_j y_j + shared(x)

The expert bias b gets no gradient (noaux_tc balances load with a separate
update rule, which the pages do not print; balance.py holds the reading of
it that the library implements).
"""
from __future__ import annotations

import numpy as np


def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def _silu(z):
    return z * _sigmoid(z)


def _dsilu(z):
    sg = _sigmoid(z)
    return sg * (1.0 + z * (1.0 - sg))


def forward(x, wg, w13, w2, w13s, w2s, idx, norm_topk_prob=True, rsf=1.0):
    """fp64 forward pass on fp64 arrays for a fixed choice `idx` [T, k].

    Shapes: x [T, H], wg [E, H], w13 [E, 2I, H] (gate rows then up rows),
    w2 [E, H, I], w13s [2Is, H], w2s [H, Is] (Is may be 0: w13s/w2s None).
    Returns (out [T, H], cache) with the intermediates the backward pass uses."""
    T, H = x.shape
    E, I2, _ = w13.shape
    I = I2 // 2
    k = idx.shape[1]
    L = x @ wg.T
    s = _sigmoid(L)
    ssel = np.take_along_axis(s, idx, 1)
    S = ssel.sum(1, keepdims=True)
    w = rsf * (ssel / S if norm_topk_prob else ssel)
    out = np.zeros((T, H))
    g = np.zeros((T, k, I))
    u = np.zeros((T, k, I))
    y = np.zeros((T, k, H))
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            g[t, j] = w13[e, :I] @ x[t]
            u[t, j] = w13[e, I:] @ x[t]
            y[t, j] = w2[e] @ (_silu(g[t, j]) * u[t, j])
            out[t] += w[t, j] * y[t, j]
    gs = us = None
    if w13s is not None:
        Is = w13s.shape[0] // 2
        gs = x @ w13s[:Is].T
        us = x @ w13s[Is:].T
        out += (_silu(gs) * us) @ w2s.T
    cache = dict(L=L, s=s, ssel=ssel, S=S, w=w, g=g, u=u, y=y, gs=gs, us=us)
    return out, cache


def backward(x, wg, w13, w2, w13s, w2s, idx, dout, norm_topk_prob=True, rsf=1.0):
    """Gradients of sum(out * dout) with the choice `idx` held fixed.

    Returns a dict: dx [T, H], dwg [E, H], dw13 [E, 2I, H], dw2 [E, H, I],
    dw13s, dw2s (None without a shared expert), dw [T, k] (routing weights),
    dlogits [T, E] (zero off the chosen experts)."""
    out, c = forward(x, wg, w13, w2, w13s, w2s, idx, norm_topk_prob, rsf)
    T, H = x.shape
    E, I2, _ = w13.shape
    I = I2 // 2
    k = idx.shape[1]
    dx = np.zeros_like(x)
    dw13 = np.zeros_like(w13)
    dw2 = np.zeros_like(w2)
    dw = np.zeros((T, k))
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            g, u = c["g"][t, j], c["u"][t, j]
            a = _silu(g) * u
            # out += w * y  ->  dw = <dout, y>,  dy = w * dout
            dw[t, j] = dout[t] @ c["y"][t, j]
            dy = c["w"][t, j] * dout[t]
            # y = W2 a  ->  da = W2^T dy,  dW2 += dy a^T
            da = w2[e].T @ dy
            dw2[e] += np.outer(dy, a)
            # a = SiLU(g) * u
            dg = da * u * _dsilu(g)
            du = da * _silu(g)
            # g = Wgate x, u = Wup x
            dw13[e, :I] += np.outer(dg, x[t])
            dw13[e, I:] += np.outer(du, x[t])
            dx[t] += w13[e, :I].T @ dg + w13[e, I:].T @ du
    dw13s = dw2s = None
    if w13s is not None:
        Is = w13s.shape[0] // 2
        gs, us = c["gs"], c["us"]
        a = _silu(gs) * us
        dw2s = dout.T @ a
        da = dout @ w2s
        dg = da * us * _dsilu(gs)
        du = da * _silu(gs)
        dw13s = np.concatenate([dg.T @ x, du.T @ x], axis=0)
        dx += dg @ w13s[:Is] + du @ w13s[Is:]
    # routing weights -> selected sigmoid scores
    ssel, S = c["ssel"], c["S"]
    if norm_topk_prob:
        # w_j = rsf s_j / S:  ds_m = rsf (dw_m / S - sum_j dw_j s_j / S^2)
        dssel = rsf * (dw / S - (dw * ssel).sum(1, keepdims=True) / S ** 2)
    else:
        dssel = rsf * dw
    ds = np.zeros((T, E))
    np.put_along_axis(ds, idx, dssel, 1)
    # s = sigmoid(L)
    dlogits = ds * c["s"] * (1.0 - c["s"])
    dx += dlogits @ wg
    dwg = dlogits.T @ x
    return dict(out=out, dx=dx, dwg=dwg, dw13=dw13, dw2=dw2, dw13s=dw13s, dw2s=dw2s, dw=dw,
                dlogits=dlogits)


def expert_grads(x, dout, w, w13, w2):
    """Weight gradients of ONE SwiGLU expert from the rows that chose it, the
    chain rule of backward() restricted to that expert (what a full-size check
    can afford: one expert's weights, not all of them).

    x [n, H] and dout [n, H]: the rows' token inputs and upstream gradients;
    w [n]: their routing weights (1 for the shared expert, which every token
    uses); w13 [2I, H] (gate rows, then up rows), w2 [H, I].
    Returns (dw13 [2I, H], dw2 [H, I])."""
    I = w13.shape[0] // 2
    g = x @ w13[:I].T
    u = x @ w13[I:].T
    a = _silu(g) * u
    dy = w[:, None] * dout          # out += w y
    dw2 = dy.T @ a                  # y = W2 a
    da = dy @ w2
    dg = da * u * _dsilu(g)         # a = SiLU(g) u
    du = da * _silu(g)
    dw13 = np.concatenate([dg.T @ x, du.T @ x], axis=0)
    return dw13, dw2

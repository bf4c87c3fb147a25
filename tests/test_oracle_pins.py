"""Pins of the CPU oracle against facts that do not come from the oracle.

Each test checks one oracle function against a closed form, a hand-derived
fixture (tests/golden), a library routine, brute force on a tiny input, or an
invariant that the method fixes.  No GPU is used.
"""
import json
import math
import os
from fractions import Fraction
from itertools import combinations

import numpy as np
import pytest
import torch

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def ulps(a, b):
    """|a - b| in units of the binary32 spacing at b."""
    b32 = np.asarray(b, dtype=np.float32)
    return np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)) / np.spacing(
        np.abs(b32)).astype(np.float64)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def bf16_value(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- number formats

def test_exp_against_libm():
    x = np.linspace(-86, 86, 400_001, dtype=np.float32)
    y = O.exp_f32(x)
    assert ulps(y, np.exp(x.astype(np.float64))).max() <= 1.0
    assert O.exp_f32(np.float32([0.0]))[0] == 1.0


def test_exp_clamps_outside_range():
    y = O.exp_f32(np.float32([-200.0, -86.0, 86.0, 200.0]))
    assert y[0] == y[1] and y[2] == y[3]
    assert np.isfinite(y).all()


def test_sigmoid_closed_forms_and_libm():
    s = O.sigmoid_f32(np.float32([0.0, math.log(3), -math.log(3), math.log(7)]))
    assert s[0] == 0.5
    assert ulps(s[1:], [0.75, 0.25, 0.875]).max() <= 2
    x = np.linspace(-80, 80, 200_001, dtype=np.float32)
    ref = 1.0 / (1.0 + np.exp(-x.astype(np.float64)))
    assert ulps(O.sigmoid_f32(x), ref).max() <= 3
    # symmetry s(-l) = 1 - s(l) holds to rounding
    assert np.abs(O.sigmoid_f32(-x) - (1 - O.sigmoid_f32(x))).max() < 1e-6


def test_bf16_roundtrip_and_ties():
    assert O.f32_to_bf16(np.float32([1.0]))[0] == 0x3F80
    # 1 + 2^-8 lies halfway between bf16 1.0 and 1.0078125: even mantissa wins
    assert O.f32_to_bf16(np.float32([1 + 2 ** -8]))[0] == 0x3F80
    assert O.f32_to_bf16(np.float32([1 + 3 * 2 ** -8]))[0] == 0x3F82
    v = np.random.default_rng(1).standard_normal(5000).astype(np.float32) * 100
    assert (O.f32_to_bf16(v) == bf16_bits(v)).all()          # torch's RNE cast
    b = bf16_bits(v)
    assert (O.bf16_to_f32(b) == bf16_value(b)).all()


def test_e4m3_decode_all_codes_against_torch():
    codes = np.arange(256, dtype=np.uint8)
    mine = O.e4m3_to_f32(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    finite = ~np.isnan(ref)
    assert np.isnan(mine[~finite]).all()
    assert (mine[finite] == ref[finite]).all()
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9 and mine[0x38] == 1.0


def test_e4m3_encode_against_torch_and_saturation():
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.standard_normal(20000) * 10, rng.standard_normal(2000) * 1e-2,
                        rng.uniform(-440, 440, 2000)]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (O.f32_to_e4m3(v) == ref).all()
    assert O.f32_to_e4m3(np.float32([1000.0, -1e9]))[0] == 0x7E
    assert O.f32_to_e4m3(np.float32([-1e9]))[0] == 0xFE


def test_activation_quantisation_recipe():
    rng = np.random.default_rng(3)
    v = rng.standard_normal((5, 300)).astype(np.float32)
    v[2, 128:256] = 0.0
    q, s = O.quant_act_e4m3(v)
    assert s.shape == (5, 3)
    for r in range(5):
        for b in range(3):
            blk = v[r, b * 128:(b + 1) * 128]
            amax = np.float32(np.abs(blk).max())
            want = np.float32(amax / np.float32(448.0)) if amax > 0 else np.float32(1.0)
            assert s[r, b] == want
            ref = torch.from_numpy(blk / want).to(torch.float8_e4m3fn).view(torch.uint8)
            assert (q[r, b * 128:(b + 1) * 128] == ref.numpy()).all()
    assert (q[2, 128:256] == 0).all()


# ---------------------------------------------------------------- router

def _sym(v, table):
    return table[v] if isinstance(v, str) else float(v)


def _frac(s):
    return float(Fraction(s))


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "routing_closed_form.json")))["cases"],
                         ids=lambda c: c["name"])
def test_route_closed_form_fixture(case):
    table = json.load(open(os.path.join(GOLDEN, "routing_closed_form.json")))["logit_symbols"]
    E, k = case["E"], case["k"]
    cfg = O.Config(T=1, H=8, E=E, k=k, I=8, n_group=case["n_group"],
                   topk_group=case["topk_group"], group_topn=case.get("group_topn", 2))
    L = np.array([[_sym(v, table) for v in case["logits"]]], dtype=np.float32)
    idx, w, _ = O.route(cfg, L, np.array(case["bias"], dtype=np.float32))
    assert idx[0].tolist() == case["idx"]
    assert ulps(w[0], [_frac(f) for f in case["w"]]).max() <= 4


def _brute_force_route(L, b, k, G, tg, tn):
    """Exhaustive search over expert subsets on tiny inputs."""
    T, E = L.shape
    s = O.sigmoid_f32(L).astype(np.float32)
    c = (s + b[None, :]).astype(np.float32)
    gsz = E // G
    out = []
    for t in range(T):
        # groups: the admissible group sets are those whose score sum is maximal,
        # found by ranking all subsets of size tg (lexicographic tie-break by
        # descending score then lower index, as a sort key)
        if G > 1:
            gs = [np.sort(c[t, g * gsz:(g + 1) * gsz])[::-1][:tn].astype(np.float64).sum()
                  for g in range(G)]
            order = sorted(range(G), key=lambda g: (-gs[g], g))
            keep = set(order[:tg])
        else:
            keep = {0}
        elig = [e for e in range(E) if (e // gsz) in keep]
        best = None
        for sub in combinations(elig, k):
            key = sorted(((-c[t, e], e) for e in sub))
            if best is None or key < best:
                best = key
        out.append([e for _, e in best])
    return np.array(out, dtype=np.int32), s


@pytest.mark.parametrize("E,k,G,tg", [(8, 3, 1, 1), (8, 2, 4, 2), (12, 3, 3, 2), (6, 6, 1, 1)])
def test_route_brute_force_tiny(E, k, G, tg):
    rng = np.random.default_rng(E * 100 + k)
    T = 40
    L = (rng.standard_normal((T, E)) * 1.5).astype(np.float32)
    b = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    cfg = O.Config(T=T, H=8, E=E, k=k, I=8, n_group=G, topk_group=tg, group_topn=2)
    idx, w, _ = O.route(cfg, L, b)
    bidx, s = _brute_force_route(L, b, k, G, tg, 2)
    assert (idx == bidx).all()
    sel = np.take_along_axis(s.astype(np.float64), idx, axis=1)
    assert np.allclose(w, sel / sel.sum(1, keepdims=True), rtol=4e-7, atol=0)


def test_route_invariants_dots3_shape():
    rng = np.random.default_rng(7)
    T, E, k = 512, 256, 8
    L = (rng.standard_normal((T, E)) * 1.43).astype(np.float32)
    b = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    cfg = O.Config(T=T, H=8, E=E, k=k, I=8)
    idx, w, gap = O.route(cfg, L, b)
    # k distinct experts per token, weights summing to 1
    assert all(len(set(r)) == k for r in idx.tolist())
    assert np.abs(w.astype(np.float64).sum(1) - 1).max() < k * 2 ** -23
    # keys are non-increasing along the slots
    c = O.sigmoid_f32(L) + b
    ck = np.take_along_axis(c, idx, 1)
    assert (np.diff(ck, axis=1) <= 0).all()
    # the bias only steers: weights equal renormalised unbiased scores
    s = np.take_along_axis(O.sigmoid_f32(L).astype(np.float64), idx, 1)
    assert np.allclose(w, s / s.sum(1, keepdims=True), rtol=4e-7, atol=0)
    # relabelling experts (logits and bias together) relabels the choice
    perm = rng.permutation(E)
    idx2, w2, _ = O.route(cfg, L[:, perm], b[perm])
    clear = gap > 1e-4
    assert (perm[idx2][clear] == idx[clear]).all()
    assert (w2[clear] == w[clear]).all()
    # a constant bias shift keeps the choice away from near-ties
    idx3, _, _ = O.route(cfg, L, b + np.float32(0.25))
    assert (idx3[clear] == idx[clear]).all()


def test_route_zero_bias_is_topk_of_logits_and_bias_concentrates_decode_load():
    """With b = 0 the choice is the k largest logits (sigmoid is increasing;
    equal logits by lower index), i.e. a stable argsort.  With the decode
    batch's U(-0.1, 0.1) bias the same 64 tokens touch far fewer experts: their
    top-8 sigmoid scores lie close together near 1, so the bias decides."""
    T, E, k = 64, 256, 8
    cfg = O.Config(T=T, H=8, E=E, k=k, I=8)
    for seed in range(3):
        rng = np.random.default_rng(seed)
        L = (rng.standard_normal((T, E)) * 1.43).astype(np.float32)
        b = rng.uniform(-0.1, 0.1, E).astype(np.float32)
        idx0, w0, _ = O.route(cfg, L, np.zeros(E, np.float32))
        assert (idx0 == np.argsort(-L, axis=1, kind="stable")[:, :k]).all()
        idx1, _, _ = O.route(cfg, L, b)
        touched0, touched1 = len(np.unique(idx0)), len(np.unique(idx1))
        # a uniform choice of 8 of 256 for 64 tokens touches ~221 on average
        assert 205 <= touched0 <= 240
        assert touched1 <= 170


def test_route_forced_selection_weights_do_not_see_bias():
    rng = np.random.default_rng(8)
    T, E, k = 64, 32, 4
    L = rng.standard_normal((T, E)).astype(np.float32)
    b = np.zeros(E, np.float32)
    forced = [3, 17, 20, 31]
    b[forced] = 10.0
    cfg = O.Config(T=T, H=8, E=E, k=k, I=8)
    idx, w, _ = O.route(cfg, L, b)
    assert all(sorted(r) == forced for r in idx.tolist())
    s = O.sigmoid_f32(L).astype(np.float64)
    for t in range(T):
        sel = s[t, idx[t]]
        assert np.allclose(w[t], sel / sel.sum(), rtol=4e-7, atol=0)


def test_route_without_renormalisation_and_scaling():
    rng = np.random.default_rng(9)
    L = rng.standard_normal((16, 16)).astype(np.float32)
    b = np.zeros(16, np.float32)
    cfg = O.Config(T=16, H=8, E=16, k=3, I=8, norm_topk_prob=False, routed_scaling_factor=2.5)
    idx, w, _ = O.route(cfg, L, b)
    s = np.take_along_axis(O.sigmoid_f32(L), idx, 1)
    assert (w == (s * np.float32(2.5)).astype(np.float32)).all()


def test_route_rejects_bad_configs():
    L = np.zeros((1, 8), np.float32)
    b = np.zeros(8, np.float32)
    for kw in ({"k": 9}, {"n_group": 3}, {"n_group": 4, "topk_group": 5}, {"k": 0}):
        args = dict(T=1, H=8, E=8, k=2, I=8)
        args.update(kw)
        with pytest.raises(ValueError):
            O.route(O.Config(**args), L, b)


def test_router_logits_against_matmul():
    rng = np.random.default_rng(10)
    T, H, E = 24, 96, 16
    x = bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    wg = bf16_bits((rng.standard_normal((E, H)) * 0.02).astype(np.float32))
    cfg = O.Config(T=T, H=H, E=E, k=2, I=8)
    ref = bf16_value(x) @ bf16_value(wg).T
    assert np.allclose(O.router_logits(cfg, x, wg), ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- permute

@pytest.mark.parametrize("T,E,k", [(1, 4, 1), (37, 8, 3), (256, 256, 8), (100, 32, 32)])
def test_permute_against_stable_argsort(T, E, k):
    rng = np.random.default_rng(T + E)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    cfg = O.Config(T=T, H=8, E=E, k=k, I=8)
    offsets, rows, pos = O.permute(cfg, idx)
    flat = idx.ravel()
    order = np.argsort(flat, kind="stable")
    assert (offsets == np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))])).all()
    assert (rows == order // k).all()
    assert (pos[order] == np.arange(T * k)).all()
    assert (np.diff(offsets) >= 0).all() and offsets[-1] == T * k


# ---------------------------------------------------------------- layer

def _rand_bits(rng, shape, std):
    return bf16_bits((rng.standard_normal(shape) * std).astype(np.float32))


def _silu(g):
    return g / (1.0 + np.exp(-g))


def _dense_masked_layer(cfg, x, idx, w, w13, w2, w13s, w2s):
    """Every expert on every token, then a {0, w} mask: no dispatch at all."""
    X = bf16_value(x)
    T, E, I, H = cfg.T, cfg.E, cfg.I, cfg.H
    mask = np.zeros((T, E))
    for t in range(T):
        for j in range(cfg.k):
            mask[t, idx[t, j]] += float(w[t, j])
    out = np.zeros((T, H))
    for e in range(E):
        W13 = bf16_value(w13[e])
        Ye = (_silu(X @ W13[:I].T) * (X @ W13[I:].T)) @ bf16_value(w2[e]).T
        out += mask[:, e:e + 1] * Ye
    Is = cfg.n_shared * I
    if Is:
        W13s = bf16_value(w13s)
        out += (_silu(X @ W13s[:Is].T) * (X @ W13s[Is:].T)) @ bf16_value(w2s).T
    return out


@pytest.mark.parametrize("E,k,S", [(8, 2, 1), (6, 6, 2), (8, 1, 0)])
def test_layer_against_dense_masked_brute_force(E, k, S):
    rng = np.random.default_rng(E * 10 + k)
    T, H, I = 12, 48, 16
    cfg = O.Config(T=T, H=H, E=E, k=k, I=I, n_shared=S)
    x = _rand_bits(rng, (T, H), 1.0)
    wg = _rand_bits(rng, (E, H), 0.2)
    w13 = _rand_bits(rng, (E, 2 * I, H), 0.2)
    w2 = _rand_bits(rng, (E, H, I), 0.2)
    w13s = _rand_bits(rng, (2 * S * I, H), 0.2)
    w2s = _rand_bits(rng, (H, S * I), 0.2)
    L = O.router_logits(cfg, x, wg).astype(np.float32)
    idx, w, _ = O.route(cfg, L, rng.uniform(-0.1, 0.1, E).astype(np.float32))
    got = O.layer(cfg, x, idx, w, w13, w2, w13s, w2s)
    ref = _dense_masked_layer(cfg, x, idx, w, w13, w2, w13s, w2s)
    assert np.allclose(got, ref, rtol=1e-10, atol=1e-10)


def _perm_matrix_bits(perm):
    n = len(perm)
    m = np.zeros((n, n), np.float32)
    m[np.arange(n), perm] = 1.0
    return bf16_bits(m)


def test_layer_permutation_matrix_closed_form():
    """Gate, up and down set to permutation matrices: y = P3 (SiLU(P1 x) * P2 x),
    i.e. y[h] = SiLU(x[p1[p3[h]]]) * x[p2[p3[h]]] by index arithmetic alone.
    A transposed operand would use the inverse permutation and fail."""
    rng = np.random.default_rng(11)
    T, H, E, k = 6, 16, 4, 2
    I = H
    cfg = O.Config(T=T, H=H, E=E, k=k, I=I, n_shared=1)
    x = _rand_bits(rng, (T, H), 1.0)
    X = bf16_value(x)
    perms = [[rng.permutation(H) for _ in range(3)] for _ in range(E + 1)]
    w13 = np.stack([np.concatenate([_perm_matrix_bits(p[0]), _perm_matrix_bits(p[1])])
                    for p in perms[:E]])
    w2 = np.stack([_perm_matrix_bits(p[2]) for p in perms[:E]])
    ps = perms[E]
    w13s = np.concatenate([_perm_matrix_bits(ps[0]), _perm_matrix_bits(ps[1])])
    w2s = _perm_matrix_bits(ps[2])
    idx = np.array([rng.permutation(E)[:k] for _ in range(T)], np.int32)
    w = rng.uniform(0.1, 1.0, (T, k)).astype(np.float32)
    got = O.layer(cfg, x, idx, w, w13, w2, w13s, w2s)

    def expert(p, xt):
        return np.array([_silu(xt[p[0][p[2][h]]]) * xt[p[1][p[2][h]]] for h in range(H)])

    for t in range(T):
        want = expert(ps, X[t]) + sum(float(w[t, j]) * expert(perms[idx[t, j]], X[t])
                                      for j in range(k))
        assert np.allclose(got[t], want, rtol=1e-12, atol=1e-12)


def test_layer_special_cases():
    rng = np.random.default_rng(12)
    T, H, E, k, I = 8, 32, 4, 4, 8
    cfg = O.Config(T=T, H=H, E=E, k=k, I=I, n_shared=1)
    w13 = _rand_bits(rng, (E, 2 * I, H), 0.3)
    w2 = _rand_bits(rng, (E, H, I), 0.3)
    w13s = _rand_bits(rng, (2 * I, H), 0.3)
    w2s = _rand_bits(rng, (H, I), 0.3)
    wg = _rand_bits(rng, (E, H), 0.3)
    # x = 0: every expert output is SiLU(0) * 0 = 0
    x0 = np.zeros((T, H), np.uint16)
    L0 = O.router_logits(cfg, x0, wg).astype(np.float32)
    assert (L0 == 0).all()
    idx0, w0, _ = O.route(cfg, L0, rng.uniform(-0.1, 0.1, E).astype(np.float32))
    assert np.allclose(w0, 1.0 / k)
    assert (O.layer(cfg, x0, idx0, w0, w13, w2, w13s, w2s) == 0).all()
    # k = E: every expert chosen, so the bias cannot change the output
    x = _rand_bits(rng, (T, H), 1.0)
    L = O.router_logits(cfg, x, wg).astype(np.float32)
    outs = []
    for bias in (np.zeros(E, np.float32), rng.uniform(-1, 1, E).astype(np.float32)):
        idx, w, _ = O.route(cfg, L, bias)
        outs.append(O.layer(cfg, x, idx, w, w13, w2, w13s, w2s))
    # the bias reorders the slots, so the binary32 weight sum is rounded in a
    # different order: equal up to binary32 rounding of the weights
    assert np.allclose(outs[0], outs[1], rtol=2e-6, atol=1e-7)
    # routed_scaling_factor 0 leaves the shared expert alone
    cfg0 = O.Config(T=T, H=H, E=E, k=2, I=I, n_shared=1, routed_scaling_factor=0.0)
    idx, w, _ = O.route(cfg0, L, np.zeros(E, np.float32))
    assert (w == 0).all()
    shared_only = O.layer(cfg0, x, idx, w, w13, w2, w13s, w2s)
    X = bf16_value(x)
    W13s = bf16_value(w13s)
    ref = (_silu(X @ W13s[:I].T) * (X @ W13s[I:].T)) @ bf16_value(w2s).T
    assert np.allclose(shared_only, ref, rtol=1e-10, atol=1e-12)
    # token independence: a subset of tokens gives the same rows
    idx, w, _ = O.route(cfg, L, np.zeros(E, np.float32))
    full = O.layer(cfg, x, idx, w, w13, w2, w13s, w2s)
    sub = O.layer(cfg, x, idx, w, w13, w2, w13s, w2s, tokens=np.array([5, 1], np.int32))
    assert (sub == full[[5, 1]]).all()


def test_layer_fp8_against_dense_dequantised_brute_force():
    """fp8 mode: weights are e4m3 codes times 128x128 block scales, and each
    GEMM's activation operand goes through the per-128 e4m3 recipe.  Checked
    with torch's e4m3 cast doing the quantisation."""
    rng = np.random.default_rng(13)
    T, H, E, k, I = 5, 256, 3, 2, 128
    cfg = O.Config(T=T, H=H, E=E, k=k, I=I, n_shared=1, fp8=True)

    def qweight(shape):
        w = (rng.standard_normal(shape) * 0.05).astype(np.float32)
        R, C = shape
        q = np.empty(shape, np.uint8)
        s = np.empty((R // 128, C // 128), np.float32)
        for i in range(R // 128):
            for j in range(C // 128):
                blk = w[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
                s[i, j] = np.abs(blk).max() / np.float32(448)
                q[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128] = torch.from_numpy(
                    blk / s[i, j]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        return q, s

    def deq(q, s):
        v = torch.from_numpy(q).view(torch.float8_e4m3fn).double().numpy()
        return v * np.kron(s.astype(np.float64), np.ones((128, 128)))

    def qact(v):  # per row, per 128 columns
        out = np.empty_like(v)
        for r in range(v.shape[0]):
            for b in range(v.shape[1] // 128):
                blk = v[r, b * 128:(b + 1) * 128].astype(np.float32)
                amax = np.float32(np.abs(blk).max())
                sc = np.float32(amax / np.float32(448)) if amax > 0 else np.float32(1)
                q = torch.from_numpy(blk / sc).to(torch.float8_e4m3fn).double().numpy()
                out[r, b * 128:(b + 1) * 128] = q * np.float64(sc)
        return out

    x = _rand_bits(rng, (T, H), 1.0)
    w13 = [qweight((2 * I, H)) for _ in range(E)]
    w2 = [qweight((H, I)) for _ in range(E)]
    w13s, w2s = qweight((2 * I, H)), qweight((H, I))
    idx = np.array([rng.permutation(E)[:k] for _ in range(T)], np.int32)
    w = rng.uniform(0.1, 1.0, (T, k)).astype(np.float32)
    got = O.layer(cfg, x, idx, w, np.stack([q for q, _ in w13]), np.stack([q for q, _ in w2]),
                  w13s[0], w2s[0], w13_scale=np.stack([s for _, s in w13]),
                  w2_scale=np.stack([s for _, s in w2]), w13s_scale=w13s[1], w2s_scale=w2s[1])
    Xq = qact(bf16_value(x))

    def ffn(p13, p2):
        W13 = deq(*p13)
        A = _silu(Xq @ W13[:I].T) * (Xq @ W13[I:].T)
        return qact(A) @ deq(*p2).T

    ref = ffn(w13s, w2s)
    for e in range(E):
        Ye = ffn(w13[e], w2[e])
        m = np.array([float(w[t, list(idx[t]).index(e)]) if e in idx[t] else 0.0
                      for t in range(T)])
        ref += m[:, None] * Ye
    # A is quantised from its fp32 rounding in the oracle and from fp64 here:
    # a code can move by one step at a rounding boundary, hence the tolerance
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-3


# ---------------------------------------------------------------- pre-norm block
def _bf16_value(b):
    return float(np.array([int(b) << 16], dtype=np.uint32).view(np.float32)[0])


def _nearest_bf16_exact(d: float) -> int:
    """Brute force: the bf16 pattern nearest to d in exact rational arithmetic,
    ties to the even pattern (independent of the oracle's scaling method)."""
    x = Fraction(d)
    f = np.array([d], dtype=np.float32).view(np.uint32)[0] >> 16  # a nearby pattern
    best = None
    for c in range(int(f) - 2, int(f) + 3):
        c &= 0xFFFF
        v = _bf16_value(c)
        if not math.isfinite(v):
            continue
        err = abs(Fraction(v) - x)
        key = (err, c & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


def test_f64_to_bf16_is_nearest_even():
    rng = np.random.default_rng(7)
    vals = list(rng.standard_normal(300) * 10.0 ** rng.integers(-30, 30, 300))
    vals += [1.0 + 2.0 ** -8, 1.0 + 2.0 ** -8 + 2.0 ** -40, 1.0 + 3 * 2.0 ** -8,
             -(1.0 + 2.0 ** -8), 2.0 ** -130, 3 * 2.0 ** -134, 2.0 ** -127 * 1.5]
    got = O.f64_to_bf16(np.array(vals))
    for d, g in zip(vals, got):
        assert int(g) == _nearest_bf16_exact(d), (d, hex(int(g)))
    assert int(O.f64_to_bf16(np.array([1e39]))[0]) == 0x7F80
    assert int(O.f64_to_bf16(np.array([-0.0]))[0]) == 0x8000


def test_rmsnorm_closed_forms():
    H = 64
    one = np.full(H, 0x3F80, dtype=np.uint16)
    two = np.full(H, 0x4000, dtype=np.uint16)
    # constant row c: u = gamma * c / sqrt(c^2 + eps)
    c = O.f32_to_bf16(np.array([3.0], dtype=np.float32))[0]
    h = np.full((1, H), c, dtype=np.uint16)
    u, r = O.rmsnorm(h, two, 1e-6)
    exp_u = _nearest_bf16_exact(2.0 * 3.0 / math.sqrt(9.0 + 1e-6))
    assert (u == exp_u).all() and abs(r[0] - 1.0 / math.sqrt(9.0 + 1e-6)) < 1e-15
    # one non-zero entry v in a row of H: mean square v^2 / H, so u = sqrt(H) sign(v)
    h = np.zeros((1, H), dtype=np.uint16)
    h[0, 5] = O.f32_to_bf16(np.array([-0.75], dtype=np.float32))[0]
    u, _ = O.rmsnorm(h, one, 0.0)
    assert _bf16_value(u[0, 5]) == -8.0 and (np.delete(u[0], 5) == 0).all()
    # eps-dominated rows: |h| << sqrt(eps) gives u ~ h / sqrt(eps)
    h = np.full((1, H), O.f32_to_bf16(np.array([1e-6], dtype=np.float32))[0], dtype=np.uint16)
    hv = _bf16_value(h[0, 0])
    u, _ = O.rmsnorm(h, one, 1e-6)
    assert int(u[0, 0]) == _nearest_bf16_exact(hv / math.sqrt(hv * hv + 1e-6))


def test_rmsnorm_invariants():
    rng = np.random.default_rng(3)
    T, H = 6, 256
    h = O.f32_to_bf16(rng.standard_normal((T, H)).astype(np.float32))
    g1 = np.full(H, 0x3F80, dtype=np.uint16)
    u, _ = O.rmsnorm(h, g1, 0.0)
    uv = (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    # unit mean square up to bf16 rounding
    assert np.abs((uv ** 2).mean(axis=1) - 1.0).max() < 4e-3
    # exact invariance under a power-of-two rescale of the row (eps = 0)
    h2 = O.f32_to_bf16(((h.astype(np.uint32) << 16).view(np.float32) * 8.0).astype(np.float32))
    u2, _ = O.rmsnorm(h2, g1, 0.0)
    assert (u2 == u).all()
    # gamma scales the output column-wise (a power of two: exact)
    g4 = np.full(H, 0x4080, dtype=np.uint16)  # 4.0
    u4, _ = O.rmsnorm(h, g4, 0.0)
    assert np.array_equal((u4.astype(np.uint32) << 16).view(np.float32),
                          4.0 * (u.astype(np.uint32) << 16).view(np.float32))


def test_block_is_residual_plus_layer():
    rng = np.random.default_rng(11)
    cfg = O.Config(T=5, H=128, E=32, k=2, I=64, n_shared=1)
    h = O.f32_to_bf16(rng.standard_normal((cfg.T, cfg.H)).astype(np.float32))
    gamma = O.f32_to_bf16((1.0 + 0.1 * rng.standard_normal(cfg.H)).astype(np.float32))
    w13 = O.f32_to_bf16((0.05 * rng.standard_normal((cfg.E, 2 * cfg.I, cfg.H))).astype(np.float32))
    w2 = O.f32_to_bf16((0.05 * rng.standard_normal((cfg.E, cfg.H, cfg.I))).astype(np.float32))
    w13s = O.f32_to_bf16((0.05 * rng.standard_normal((2 * cfg.I, cfg.H))).astype(np.float32))
    w2s = O.f32_to_bf16((0.05 * rng.standard_normal((cfg.H, cfg.I))).astype(np.float32))
    idx = np.stack([rng.choice(cfg.E, cfg.k, replace=False) for _ in range(cfg.T)]).astype(np.int32)
    w = np.full((cfg.T, cfg.k), 0.5, dtype=np.float32)
    out = O.block(cfg, h, gamma, 1e-6, idx, w, w13, w2, w13s, w2s)
    u, _ = O.rmsnorm(h, gamma, 1e-6)
    hv = (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    np.testing.assert_array_equal(out, hv + O.layer(cfg, u, idx, w, w13, w2, w13s, w2s))
    # zero expert weights: the block returns its input exactly
    z13, z2 = np.zeros_like(w13), np.zeros_like(w2)
    out0 = O.block(cfg, h, gamma, 1e-6, idx, w, z13, z2, np.zeros_like(w13s), np.zeros_like(w2s))
    np.testing.assert_array_equal(out0, hv)


# ---------------------------------------------------------------- DSA indexer
def _bf16_bits(a):
    return O.f32_to_bf16(np.asarray(a, dtype=np.float32))


def _bits_f64(b):
    return (np.asarray(b, np.uint32) << 16).view(np.float32).astype(np.float64)


def test_dsa_scores_against_einsum_and_closed_form():
    rng = np.random.default_rng(21)
    Sq, Sk, nh, D = 7, 11, 3, 16
    q = _bf16_bits(rng.standard_normal((Sq, nh, D)))
    k = _bf16_bits(rng.standard_normal((Sk, nh, D)))
    w = _bf16_bits(rng.standard_normal((Sq, nh)))
    got = O.dsa_scores(q, k, w)
    dots = np.einsum("thd,shd->tsh", _bits_f64(q), _bits_f64(k))
    ref = np.einsum("tsh,th->ts", np.maximum(dots, 0.0), _bits_f64(w))
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    # one head of width one, unit weight: I[t, s] = max(0, q_t k_s)
    q1 = _bf16_bits([[[2.0]], [[-1.5]]])
    k1 = _bf16_bits([[[3.0]], [[-4.0]], [[0.5]]])
    w1 = _bf16_bits([[1.0], [1.0]])
    np.testing.assert_array_equal(O.dsa_scores(q1, k1, w1),
                                  [[6.0, 0.0, 1.0], [0.0, 6.0, 0.0]])


def test_dsa_scores_invariants():
    rng = np.random.default_rng(22)
    Sq, Sk, nh, D = 5, 9, 4, 8
    q = _bf16_bits(rng.standard_normal((Sq, nh, D)))
    k = _bf16_bits(rng.standard_normal((Sk, nh, D)))
    w = _bf16_bits(rng.standard_normal((Sq, nh)))
    base = O.dsa_scores(q, k, w)
    # exact linearity in a power-of-two scale of the head weights
    w2 = _bf16_bits(_bits_f64(w) * 2.0)
    np.testing.assert_array_equal(O.dsa_scores(q, k, w2), 2.0 * base)
    # relabelling the heads (q, k and w together) changes nothing but summation order
    perm = rng.permutation(nh)
    np.testing.assert_allclose(O.dsa_scores(q[:, perm], k[:, perm], w[:, perm]), base,
                               rtol=1e-12, atol=1e-12)
    # ReLU: keys anti-aligned with every query in head 0 add nothing through head 0
    kneg = k.copy()
    kneg[:, 0, :] = _bf16_bits(-np.abs(_bits_f64(k[:, 0, :])))
    qpos = q.copy()
    qpos[:, 0, :] = _bf16_bits(np.abs(_bits_f64(q[:, 0, :])))
    wz = w.copy()
    wz[:, 0] = 0
    np.testing.assert_allclose(O.dsa_scores(qpos, kneg, w), O.dsa_scores(qpos, kneg, wz),
                               rtol=0, atol=0)
    # causal mask: exactly the keys past each query's absolute position are -inf
    m = O.dsa_scores(q, k, w, causal=True, q_offset=3)
    t, s = np.meshgrid(np.arange(Sq), np.arange(Sk), indexing="ij")
    assert np.isneginf(m[s > t + 3]).all() and np.isfinite(m[s <= t + 3]).all()
    np.testing.assert_array_equal(m[s <= t + 3], base[s <= t + 3])


def test_dsa_topk_against_sorted_brute_force():
    rng = np.random.default_rng(23)
    Sq, Sk, topk = 6, 40, 9
    sc = rng.integers(-3, 4, size=(Sq, Sk)).astype(np.float32)  # many ties
    sc[0, :35] = -np.inf                                        # 5 valid keys < topk
    sc[1, 7] = np.nan
    got = O.dsa_topk(sc, topk)
    for t in range(Sq):
        valid = [s for s in range(Sk) if np.isfinite(sc[t, s]) or sc[t, s] == np.inf]
        order = sorted(valid, key=lambda s: (-float(sc[t, s]), s))[:topk]
        order += [-1] * (topk - len(order))
        assert list(got[t]) == order, (t, list(got[t]), order)

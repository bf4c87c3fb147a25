"""GPU parity of the noaux_tc expert-bias update (moe_bias_update, through
the C ABI) against the reference oracle/balance.py: the updated fp32 bias
must be bit-identical (an integer histogram, an exact comparison with the
mean and one fp32 addition per expert leave no rounding choice).

Batches: random choices at several shapes, the choices the library's own
selection makes from N(0, 0.02^2 H) logits with the stored Zipf-skew bias of
the prefill workload (segment sizes from thousands of slots down to a few),
perfectly balanced loads (no change), k = 1, E = 1024, indices outside
[0, E) (counted for no expert), T = 0, gamma = 0, and three updates in a row.
"""
import numpy as np
import pytest
import torch

from oracle import balance as BAL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from sigmoid_top_routing_warp_b200 import binding
    assert torch.cuda.is_available()
    return binding


def run(B, cfg, idx, bias, gamma):
    b = torch.from_numpy(np.asarray(bias, np.float32)).cuda()
    B.moe_bias_update(cfg, torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda(), b, gamma)
    torch.cuda.synchronize()
    return b.cpu().numpy()


def random_choice(T, E, k, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("T,E,k,gamma", [(64, 256, 8, 1e-3), (300, 64, 6, 0.25), (4096, 128, 6, 1e-3),
                                         (1000, 1024, 32, 0.01), (777, 32, 1, 0.5), (50, 96, 4, 0.0)])
def test_bias_update_bit_exact_on_random_batches(B, T, E, k, gamma):
    cfg = B.MoeConfig(T=T, H=512, E=E, k=k, I=128)
    idx = random_choice(T, E, k, seed=T + E)
    bias = np.random.default_rng(E).standard_normal(E).astype(np.float32) * 0.1
    got = run(B, cfg, idx, bias, gamma)
    want = BAL.bias_update(idx, bias, gamma)
    assert (got.view(np.uint32) == want.view(np.uint32)).all()
    if gamma == 0.0:
        assert (got == bias).all()


def test_bias_update_on_the_librarys_own_skewed_choice(B):
    """The prefill workload's stored bias makes the selection's loads follow
    a capped Zipf law; three updates in a row, each on the same choice."""
    from sigmoid_top_routing_warp_b200 import workloads as W
    wl = W.WORKLOADS["prefill"]
    cfg = B.MoeConfig(T=wl.T, H=wl.H, E=wl.E, k=wl.k, I=wl.I)
    g = torch.Generator().manual_seed(5)
    logits = (torch.randn((wl.T, wl.E), generator=g) * (0.02 * wl.H ** 0.5)).float().cuda()
    route_bias = W.load_bias_table(W.bias_table_path(wl)).float().cuda()
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    B.moe_route_from_logits(cfg, logits, route_bias, idx, w)
    torch.cuda.synchronize()
    idx_h = idx.cpu().numpy()
    loads = BAL.expert_loads(idx_h, wl.E)
    assert loads.max() > 10 * loads.mean() and loads.min() < loads.mean() / 4  # skewed
    b = torch.zeros(wl.E, dtype=torch.float32, device="cuda")
    want = np.zeros(wl.E, np.float32)
    for _ in range(3):
        B.moe_bias_update(cfg, idx, b, 1e-3)
        want = BAL.bias_update(idx_h, want, 1e-3)
    torch.cuda.synchronize()
    assert (b.cpu().numpy().view(np.uint32) == want.view(np.uint32)).all()


def test_balanced_batch_and_out_of_range_indices(B):
    E, k = 64, 4
    T = 64  # every expert exactly k * T / E = 4 times
    idx = np.array([[(4 * t + j) % E for j in range(k)] for t in range(T)], np.int32)
    cfg = B.MoeConfig(T=T, H=512, E=E, k=k, I=128)
    bias = np.linspace(-1, 1, E).astype(np.float32)
    assert (run(B, cfg, idx, bias, 0.5) == bias).all()
    # indices -1 and E count for nobody (the mean still uses T * k slots)
    idx2 = idx.copy()
    idx2[0, 0], idx2[1, 1] = -1, E
    got = run(B, cfg, idx2, bias, 0.5)
    want = BAL.bias_update(idx2, bias, 0.5)
    assert (got.view(np.uint32) == want.view(np.uint32)).all()
    assert (got != bias).sum() == 2  # the two experts that lost a slot are now below the mean


def test_empty_batch_leaves_the_bias(B):
    cfg = B.MoeConfig(T=0, H=512, E=64, k=4, I=128)
    bias = np.arange(64, dtype=np.float32)
    got = run(B, cfg, np.zeros((1, 4), np.int32), bias, 1.0)
    assert (got == bias).all()

"""Pins of the expert-bias update reference (oracle/balance.py) against cases
whose answers follow from the rule by hand: equal loads, one hot expert, an
unused expert, the exact-mean tie, the fp32 addition, and invariants."""
import numpy as np
import pytest

from oracle import balance as BAL


def test_equal_loads_leave_the_bias_unchanged():
    # E = 4, k = 2, T = 4: every expert gets 2 slots = the mean
    idx = np.array([[0, 1], [2, 3], [1, 0], [3, 2]])
    b = np.array([0.5, -0.25, 0.0, 1.0], dtype=np.float32)
    assert (BAL.bias_update(idx, b, 0.125) == b).all()


def test_hand_counted_case():
    # E = 4, T = 3, k = 2: loads (3, 1, 2, 0), mean 1.5
    idx = np.array([[0, 1], [0, 2], [0, 2]])
    b = np.zeros(4, dtype=np.float32)
    got = BAL.bias_update(idx, b, 0.25)
    assert got.tolist() == [-0.25, 0.25, -0.25, 0.25]
    assert BAL.expert_loads(idx, 4).tolist() == [3, 1, 2, 0]


def test_exact_mean_is_a_tie_even_when_not_an_integer_mean():
    # E = 3, n = 6: mean 2; loads (2, 3, 1) -> (0, -g, +g)
    idx = np.array([[0, 1], [1, 2], [0, 1]])
    got = BAL.bias_update(idx, np.zeros(3, np.float32), 1.0)
    assert got.tolist() == [0.0, -1.0, 1.0]
    # E = 4, n = 6: mean 1.5, no expert can sit on it
    idx = np.array([[0, 1], [1, 2], [0, 1]])
    got = BAL.bias_update(idx, np.zeros(4, np.float32), 1.0)
    assert got.tolist() == [-1.0, -1.0, 1.0, 1.0]


def test_update_is_one_fp32_addition():
    # 1 + 2^-30 is not representable in fp32: the raised bias stays 1.0
    idx = np.array([[1]])
    b = np.array([1.0, 1.0], dtype=np.float32)
    got = BAL.bias_update(idx, b, 2.0 ** -30)
    assert got.dtype == np.float32 and got.tolist() == [1.0, 1.0]
    # 2^-24 below 1 is representable: the lowered expert moves, the raised one rounds back
    got = BAL.bias_update(idx, b, 2.0 ** -24)
    assert got[1] == np.float32(1.0) - np.float32(2.0 ** -24) and got[0] == 1.0


def test_empty_batch_and_out_of_range_indices():
    b = np.array([0.1, 0.2], dtype=np.float32)
    assert (BAL.bias_update(np.zeros((0, 2), np.int64), b, 0.5) == b).all()
    # an index outside [0, E) is a slot of nobody: loads (1, 0), n = 2, mean 1
    got = BAL.bias_update(np.array([[0, 7]]), np.zeros(2, np.float32), 1.0)
    assert got.tolist() == [0.0, 1.0]


def test_invariants_on_random_batches():
    rng = np.random.default_rng(3)
    for E, T, k in ((8, 50, 2), (64, 300, 6), (256, 64, 8)):
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
        b = rng.standard_normal(E).astype(np.float32)
        g = 1e-3
        got = BAL.bias_update(idx, b, g)
        loads = BAL.expert_loads(idx, E)
        assert loads.sum() == T * k
        over, under = loads * E > T * k, loads * E < T * k
        assert (got[over] < b[over]).all() and (got[under] > b[under]).all()
        assert (got[~over & ~under] == b[~over & ~under]).all()
        # brute force on the definition, expert by expert
        for e in range(E):
            cnt = int((idx == e).sum())
            want = b[e] if cnt * E == T * k else np.float32(b[e] + np.float32(g) * np.sign(T * k / E - cnt))
            assert got[e] == np.float32(want)

"""Pins for the oracle's gate top-k and histogram (CPU only).

The oracle is checked against things it does not compute itself: brute force
by numpy's lexicographic sort, closed-form weights of hand-picked rows, the
full-softmax form of the weights, and constructed routings with known counts.
"""
import math

import numpy as np
import pytest

import oracle


def brute_topk(logits, K):
    """Full lexicographic sort on (-v, e) per row. IEEE '<' makes -0.0 and
    +0.0 equal, so they tie and fall through to the expert id."""
    N, E = logits.shape
    out = np.empty((N, K), dtype=np.int32)
    ids = np.arange(E)
    for n in range(N):
        order = np.lexsort((ids, -logits[n].astype(np.float64)))
        out[n] = order[:K]
    return out


def test_hand_row_closed_form():
    row = np.array([[0.5, 2.0, -1.0, 2.0, 0.0, -0.0]], dtype=np.float32)
    idx, w = oracle.gate_topk(row, 3)
    assert idx.tolist() == [[1, 3, 0]]
    z = 2.0 + math.exp(-1.5)
    expect = [1.0 / z, 1.0 / z, math.exp(-1.5) / z]
    np.testing.assert_allclose(w[0], expect, rtol=1e-15, atol=0)


def test_signed_zero_ties_to_lower_id():
    rows = np.array([[-0.0, 0.0, -1.0, -2.0],
                     [0.0, -0.0, -1.0, -2.0],
                     [-1.0, -0.0, -1.0, 0.0]], dtype=np.float32)
    idx, w = oracle.gate_topk(rows, 2)
    assert idx.tolist() == [[0, 1], [0, 1], [1, 3]]
    assert np.all(w == 0.5)  # equal logits: exactly 1/K


def test_all_equal_rows_pick_lowest_ids_and_uniform_weights():
    for E, K in [(8, 3), (64, 4), (160, 8), (256, 8)]:
        rows = np.full((5, E), 0.25, dtype=np.float32)
        idx, w = oracle.gate_topk(rows, K)
        assert (idx == np.arange(K)).all()
        np.testing.assert_allclose(w, 1.0 / K, rtol=1e-15)


def test_ties_at_ends_of_row():
    E = 16
    row = np.full((1, E), -3.0, dtype=np.float32)
    row[0, 0] = 1.0
    row[0, E - 1] = 1.0
    row[0, 7] = 0.5
    idx, _ = oracle.gate_topk(row, 4)
    assert idx.tolist() == [[0, E - 1, 7, 1]]


@pytest.mark.parametrize("E,K", [(4, 1), (8, 2), (13, 5), (64, 4), (160, 8), (256, 8), (32, 32)])
def test_matches_brute_force_with_many_ties(E, K):
    rng = np.random.default_rng(E * 100 + K)
    N = 300
    # few distinct values (and both zeros) so ties are common
    vals = np.array([-2.0, -1.0, -0.0, 0.0, 0.5, 1.0, 3.0], dtype=np.float32)
    logits = vals[rng.integers(0, len(vals), size=(N, E))]
    idx, w = oracle.gate_topk(logits, K)
    np.testing.assert_array_equal(idx, brute_topk(logits, K))
    # descending logits along k
    sel = np.take_along_axis(logits, idx, axis=1)
    assert (np.diff(sel.astype(np.float64), axis=1) <= 0).all()


@pytest.mark.parametrize("E,K", [(64, 4), (128, 8), (160, 8), (256, 8)])
def test_weights_equal_renormalised_full_softmax(E, K):
    """Softmax over all E logits, kept on the top K and renormalised, is the
    same number as the softmax over the K selected logits."""
    rng = np.random.default_rng(7 + E)
    logits = (rng.standard_normal((200, E)) * 2.0).astype(np.float32)
    idx, w = oracle.gate_topk(logits, K)
    x = logits.astype(np.float64)
    p = np.exp(x - x.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    ps = np.take_along_axis(p, idx, axis=1)
    ref = ps / ps.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(w, ref, rtol=1e-13, atol=0)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=4e-16 * K)
    assert (np.diff(w, axis=1) <= 0).all()


def test_shift_invariance_of_selection():
    rng = np.random.default_rng(3)
    logits = rng.standard_normal((100, 64)).astype(np.float32)
    idx0, w0 = oracle.gate_topk(logits, 4)
    # adding a power of two keeps the order of float32 values that stay exact
    idx1, w1 = oracle.gate_topk(logits * np.float32(4.0), 4)
    np.testing.assert_array_equal(idx0, idx1)


def test_count_constructed_uniform_routing():
    R, T, E, K = 4, 8, 16, 4
    N = R * T
    # token n picks experts (n*K + k) mod E: every expert hit exactly N*K/E times
    idx = ((np.arange(N)[:, None] * K + np.arange(K)[None, :]) % E).astype(np.int32)
    load_re, load_e = oracle.count(idx, R, T, E)
    assert (load_e == N * K // E).all()
    assert load_re.sum() == N * K
    for r in range(R):
        exp = np.bincount(idx[r * T:(r + 1) * T].ravel(), minlength=E)
        np.testing.assert_array_equal(load_re[r], exp)


def test_count_random_matches_bincount():
    rng = np.random.default_rng(11)
    R, T, E, K = 5, 37, 40, 3
    idx = np.stack([rng.permutation(E)[:K] for _ in range(R * T)]).astype(np.int32)
    load_re, load_e = oracle.count(idx, R, T, E)
    np.testing.assert_array_equal(load_e, np.bincount(idx.ravel(), minlength=E))
    np.testing.assert_array_equal(load_re.sum(axis=0), load_e)
    assert load_e.sum() == R * T * K


def test_count_rejects_out_of_range():
    idx = np.array([[0, 5]], dtype=np.int32)
    with pytest.raises(ValueError):
        oracle.count(idx, 1, 1, 4)

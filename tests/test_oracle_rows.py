"""Pins for the oracle's permute and combine (CPU only).

The permute is pinned by its definition evaluated with plain numpy fancy
indexing; the combine by exactly representable hand cases (dyadic weights,
small-integer bf16 rows), one-hot weights, and identity experts.
"""
import numpy as np

import oracle
import synth


def test_permute_definition_small():
    rng = np.random.default_rng(0)
    N, d, K = 6, 8, 2
    hidden = rng.integers(0, 1 << 16, size=(N, d), dtype=np.uint16)
    dest = rng.permutation(N * K).astype(np.int32).reshape(N, K)
    out = oracle.permute(hidden, K, dest)
    for n in range(N):
        for k in range(K):
            assert (out[dest[n, k]] == hidden[n]).all()


def test_permute_rows_matches_full_permute():
    rng = np.random.default_rng(1)
    N, d, K = 50, 16, 4
    hidden = rng.integers(0, 1 << 16, size=(N, d), dtype=np.uint16)
    dest = rng.permutation(N * K).astype(np.int32).reshape(N, K)
    full = oracle.permute(hidden, K, dest)
    rows = rng.choice(N * K, size=30, replace=False)
    np.testing.assert_array_equal(oracle.permute_rows(hidden, K, dest, rows), full[rows])


def test_combine_exact_dyadic_case():
    # y rows hold small integers (exact in bf16); weights are dyadic, so the
    # fp64 result is exact and can be written down by hand
    N, K, d = 2, 3, 4
    y_f = np.array([[1, 2, 3, 4], [-2, 0, 8, 1], [16, -4, 2, 2],
                    [5, 5, 5, 5], [0, 1, 0, -1], [3, 3, -3, -3]], dtype=np.float32)
    y = synth.f32_to_bf16_bits(y_f).reshape(N * K, d)
    dest = np.array([[2, 0, 1], [5, 3, 4]], dtype=np.int32)
    w = np.array([[0.5, 0.25, 0.25], [0.75, 0.125, 0.125]])
    out = oracle.combine(y, N, K, dest, w)
    expect0 = 0.5 * y_f[2] + 0.25 * y_f[0] + 0.25 * y_f[1]
    expect1 = 0.75 * y_f[5] + 0.125 * y_f[3] + 0.125 * y_f[4]
    np.testing.assert_array_equal(out, np.stack([expect0, expect1]))
    np.testing.assert_array_equal(out[0], [7.75, -1.5, 3.75, 2.25])


def test_combine_one_hot_weights_return_rows():
    rng = np.random.default_rng(2)
    N, K, d = 10, 4, 32
    y = synth.bf16_normal(N * K, d, 5, 1)
    dest = rng.permutation(N * K).astype(np.int32).reshape(N, K)
    w = np.zeros((N, K))
    pick = rng.integers(0, K, size=N)
    w[np.arange(N), pick] = 1.0
    out = oracle.combine(y, N, K, dest, w)
    np.testing.assert_array_equal(out, synth.bf16_bits_to_f32(y[dest[np.arange(N), pick]]))


def test_combine_identity_experts_reproduce_hidden():
    rng = np.random.default_rng(3)
    N, K, d = 40, 8, 64
    hidden = synth.bf16_normal(N, d, 6, 1)
    logits = rng.standard_normal((N, 16)).astype(np.float32)
    idx, w = oracle.gate_topk(logits, K)
    dest = rng.permutation(N * K).astype(np.int32).reshape(N, K)
    y = oracle.permute(hidden, K, dest)
    out = oracle.combine(y, N, K, dest, w)
    h = synth.bf16_bits_to_f32(hidden).astype(np.float64)
    np.testing.assert_allclose(out, h, rtol=1e-14, atol=1e-300)


def test_combine_token_subset_matches_full():
    rng = np.random.default_rng(4)
    N, K, d = 30, 2, 24
    y = synth.bf16_normal(N * K, d, 7, 1)
    dest = rng.permutation(N * K).astype(np.int32).reshape(N, K)
    w = rng.random((N, K))
    full = oracle.combine(y, N, K, dest, w)
    toks = np.array([29, 0, 7, 7])
    np.testing.assert_array_equal(oracle.combine(y, N, K, dest, w, tokens=toks), full[toks])

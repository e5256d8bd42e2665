"""Pins for the oracle's backward of permute and combine, weight sync and
gradient reduction (CPU only).

The backward pair is pinned by the adjoint identities of the two linear maps
(<dout, combine(y, w)> = sum_rows <dy, y>/... see each test) and by hand
cases; weight sync by its definition with numpy indexing; the reduction by a
dyadic hand case and by numpy's unbuffered add over the slot list.
"""
import numpy as np

import oracle
import synth


def _case(N=12, K=3, d=16, seed=0):
    rng = np.random.default_rng(seed)
    dest = rng.permutation(N * K).astype(np.int32).reshape(N, K)
    y = synth.bf16_normal(N * K, d, seed, 31)
    w = rng.random((N, K)).astype(np.float32)
    dout = rng.standard_normal((N, d)).astype(np.float32)
    return rng, dest, y, w, dout


def test_combine_backward_hand_case():
    # one token, two pairs, exact small values
    y_f = np.array([[1, 2, -4, 8], [0.5, -1, 2, 0]], dtype=np.float32)
    y = synth.f32_to_bf16_bits(y_f)
    dest = np.array([[1, 0]], dtype=np.int32)
    w = np.array([[0.25, 0.75]], dtype=np.float32)
    dout = np.array([[2, -1, 0.5, 1]], dtype=np.float32)
    dy, dw = oracle.combine_backward(dout, y, 2, dest, w)
    # rows in (token, k) order: k=0 -> dispatch row 1, k=1 -> row 0
    np.testing.assert_array_equal(dy, [0.25 * dout[0], 0.75 * dout[0]])
    np.testing.assert_array_equal(dw, [[np.dot(dout[0], y_f[1]), np.dot(dout[0], y_f[0])]])
    assert dw[0, 0] == 2 * 0.5 + -1 * -1 + 0.5 * 2 + 1 * 0


def test_combine_backward_adjoint_identities():
    """out = C(y, w) is linear in y and in w separately:
    <dout, out> = sum_rows <dy[row], y[row]> = sum_{n,k} w[n,k] * dw[n,k]."""
    rng, dest, y, w, dout = _case()
    N, K = w.shape
    out = oracle.combine(y, N, K, dest, w.astype(np.float64))
    dy, dw = oracle.combine_backward(dout, y, K, dest, w)
    yf = synth.bf16_bits_to_f32(y).astype(np.float64)
    lhs = float(np.sum(dout.astype(np.float64) * out))
    rows = dest.reshape(-1)
    mid = float(np.sum(dy * yf[rows]))
    rhs = float(np.sum(w.astype(np.float64) * dw))
    assert abs(lhs - mid) <= 1e-12 * (1 + abs(lhs))
    assert abs(lhs - rhs) <= 1e-12 * (1 + abs(lhs))


def test_combine_backward_token_subset():
    rng, dest, y, w, dout = _case(seed=3)
    dy, dw = oracle.combine_backward(dout, y, 3, dest, w)
    toks = np.array([11, 0, 4])
    dys, dws = oracle.combine_backward(dout, y, 3, dest, w, tokens=toks)
    K = 3
    np.testing.assert_array_equal(dws, dw[toks])
    np.testing.assert_array_equal(dys, dy.reshape(12, K, -1)[toks].reshape(-1, dy.shape[1]))


def test_permute_backward_adjoint_identity():
    """<dhidden, hidden> = <ddispatch, permute(hidden)> for the permute map."""
    rng, dest, y, w, dout = _case(seed=5)
    N, K = dest.shape
    hidden = synth.bf16_normal(N, 16, 5, 32)
    dd = synth.bf16_normal(N * K, 16, 5, 33)
    dh = oracle.permute_backward(dd, N, K, dest)
    disp = oracle.permute(hidden, K, dest)
    lhs = float(np.sum(dh * synth.bf16_bits_to_f32(hidden).astype(np.float64)))
    rhs = float(np.sum(synth.bf16_bits_to_f32(dd).astype(np.float64) *
                       synth.bf16_bits_to_f32(disp).astype(np.float64)))
    assert abs(lhs - rhs) <= 1e-12 * (1 + abs(lhs))


def test_permute_backward_sums_k_rows():
    dest = np.array([[2, 0], [1, 3]], dtype=np.int32)
    dd_f = np.array([[1, 2], [3, 4], [5, 6], [7, 8]], dtype=np.float32)
    dh = oracle.permute_backward(synth.f32_to_bf16_bits(dd_f), 2, 2, dest)
    np.testing.assert_array_equal(dh, [[6, 8], [10, 12]])


def test_weight_sync_definition():
    rng = np.random.default_rng(9)
    E, G, B = 6, 5, 48
    master = rng.integers(0, 256, size=(E, B), dtype=np.uint8)
    before = rng.integers(0, 256, size=(G, B), dtype=np.uint8)
    se = np.array([3, -1, 0, 3, -1], dtype=np.int32)
    out = oracle.weight_sync(se, master, before)
    for g in range(G):
        np.testing.assert_array_equal(out[g], master[se[g]] if se[g] >= 0 else before[g])


def test_grad_reduce_dyadic_hand_case():
    master = np.array([[1.0, 2.0], [0.5, -1.0], [4.0, 4.0]], dtype=np.float32)
    reps = np.array([[0.25, 0.25], [8.0, -2.0], [0.125, 1.0]], dtype=np.float32)
    se = np.array([0, -1, 0], dtype=np.int32)   # expert 0 has two replicas
    out = oracle.grad_reduce(se, reps, master)
    np.testing.assert_array_equal(out, [[1.375, 3.25], [0.5, -1.0], [4.0, 4.0]])


def test_grad_reduce_matches_numpy_add_at():
    rng = np.random.default_rng(4)
    E, G, W = 8, 12, 33
    master = rng.standard_normal((E, W)).astype(np.float32)
    reps = rng.standard_normal((G, W)).astype(np.float32)
    se = rng.integers(-1, E, size=G).astype(np.int32)
    out = oracle.grad_reduce(se, reps, master)
    ref = master.astype(np.float64).copy()
    used = se >= 0
    np.add.at(ref, se[used], reps[used].astype(np.float64))
    np.testing.assert_allclose(out, ref, rtol=1e-15, atol=1e-15)

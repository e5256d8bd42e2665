"""CPU check of the rule behind the gate's packed-key kernel (K = 8, E = 128
or 256), against the oracle's top-k.

The kernel orders a row's logits by a packed key: the float's order key
(-0.0 made +0.0 first) with its low log2(E) bits replaced by E-1-e. It takes
the first K+1 packed picks and keeps them when adjacent picks differ above
the dropped bits; other rows are selected again with full keys. The claim
pinned here: whenever that check passes, the first K packed picks are the
exact top-K in the exact order (larger value first, lower id among equals).
The check is exercised on normal rows (almost all pass), rows of exact ties
and signed zeros (none may pass), and rows of values a few ulps apart (none
pass). The rule is restated in numpy; the oracle is the reference.

"UltraEP" README, "Interface / 2. Forward and backward" (router top-k);
"What Happened" (routing from the exact probabilities).
"""
import numpy as np
import pytest

import oracle

K = 8


def order_key(v):
    v = (v.astype(np.float32) + np.float32(0.0)).view(np.uint32).astype(np.uint64)
    neg = (v >> np.uint64(31)) == 1
    return np.where(neg, (~v) & np.uint64(0xFFFFFFFF), v | np.uint64(0x80000000))


def packed_rule(logits):
    """(ids of the first K packed picks, whether the row passes the check)."""
    N, E = logits.shape
    lob = int(np.log2(E))
    key = order_key(logits)
    e = np.arange(E, dtype=np.uint64)
    hi_mask = np.uint64((0xFFFFFFFF >> lob) << lob)
    packed = (key & hi_mask) | (np.uint64(E - 1) - e)
    order = np.argsort(-packed.astype(np.int64), axis=1, kind="stable")[:, :K + 1]
    picks = np.take_along_axis(packed, order, 1)
    hi = picks >> np.uint64(lob)
    passes = (hi[:, :-1] != hi[:, 1:]).all(axis=1)
    return order[:, :K].astype(np.int32), passes


def rows(kind, N, E, rng):
    if kind == "normal":
        return rng.standard_normal((N, E)).astype(np.float32)
    if kind == "ties":
        vals = np.array([-1.0, -0.0, 0.0, 0.5, 1.0], dtype=np.float32)
        return vals[rng.integers(0, len(vals), size=(N, E))]
    steps = rng.integers(0, 300, size=(N, E)).astype(np.float64)
    return (1.0 + steps * 2.0 ** -23).astype(np.float32)


@pytest.mark.parametrize("E", [128, 256])
@pytest.mark.parametrize("kind", ["normal", "ties", "close"])
def test_rows_that_pass_the_check_have_the_exact_top_k(E, kind):
    rng = np.random.default_rng(E + len(kind))
    N = 3000
    x = rows(kind, N, E, rng)
    idx_or, _ = oracle.gate_topk(x, K)
    idx, passes = packed_rule(x)
    assert (idx[passes] == idx_or[passes]).all()
    if kind == "normal":
        assert passes.mean() > 0.99        # the exact re-selection is rare
    else:
        assert not passes.any()            # equal or near-equal leaders always re-select


def test_a_tie_across_the_dropped_bits_fails_the_check():
    """Two logits equal above the dropped bits but different below them: the
    packed order would put the lower id first even when its value is smaller,
    so the check must send the row to the exact path."""
    E = 128
    x = np.full((1, E), -5.0, dtype=np.float32)
    # two positive floats inside one aligned block of 128 ulps (bits
    # 0x3FC00000..0x3FC0007F), so they agree above the 7 dropped bits
    big = np.array([0x3FC00040], dtype=np.uint32).view(np.float32)[0]
    smaller = np.array([0x3FC00001], dtype=np.uint32).view(np.float32)[0]
    x[0, 3] = smaller                                  # lower id, smaller value
    x[0, 90] = big
    idx_or, _ = oracle.gate_topk(x, K)
    assert idx_or[0, 0] == 90 and idx_or[0, 1] == 3
    idx, passes = packed_rule(x)
    assert not passes[0]
    assert idx[0, 0] == 3                              # the packed order alone is wrong here

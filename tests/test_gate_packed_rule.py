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

The kernel does not sort a row: each of the warp's 32 lanes holds E/32 keys
and keeps a short sorted list of them, and each of the K+1 rounds takes the
largest list head (one warp reduction) and pops it. The lists are three deep;
a lane holding at most three keys keeps all of them and a pop fills its
bottom with 0. Otherwise a pop leaves the last entry in place, so a lane that
runs out before the last round repeats a pick, which the same adjacency check
rejects. That procedure is restated lane by lane below and checked the same
way, for every E the kernel takes (64 to 256), including rows whose leading
values sit in one lane.

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


def lane_experts(E, lane):
    """Experts lane `lane` holds: 128 c + 4 lane + j per 16-byte chunk c, then
    128 C + 32 t + lane per 4-byte tail load t."""
    nch, nt = E // 128, (E % 128) // 32
    ids = [128 * c + 4 * lane + j for c in range(nch) for j in range(4)]
    return ids + [128 * nch + 32 * t + lane for t in range(nt)]


def lane_list_rule(logits):
    """The kernel's selection, lane by lane: (ids of the first K picks, whether
    the row passes the adjacency check)."""
    N, E = logits.shape
    lob = 7 if E <= 128 else 8
    hi_mask = (0xFFFFFFFF >> lob) << lob
    vpl = E // 32
    depth = min(vpl, 3)
    fill = depth == vpl
    keys = order_key(logits).astype(np.int64)
    lanes = [np.array(lane_experts(E, l)) for l in range(32)]
    ids = np.zeros((N, K), np.int32)
    passes = np.zeros(N, bool)
    for n in range(N):
        lists = []
        for ex in lanes:
            packed = sorted(((int(keys[n, e]) & hi_mask) | (E - 1 - int(e)) for e in ex),
                            reverse=True)
            lists.append(packed[:depth])
        picks = []
        for k in range(K + 1):
            m = max(L[0] for L in lists)
            picks.append(m)
            if k == K:
                break
            for L in lists:
                if L[0] == m:
                    L[:depth - 1] = L[1:depth]
                    if fill:
                        L[depth - 1] = 0
        hi = [x >> lob for x in picks]
        passes[n] = all(hi[k] != hi[k + 1] for k in range(K))
        ids[n] = [E - 1 - (x & ((1 << lob) - 1)) for x in picks[:K]]
    return ids, passes


def clustered(N, E, rng):
    """Rows whose three to five leading values sit in one lane (all of the
    lane's values when it holds fewer)."""
    x = rng.standard_normal((N, E)).astype(np.float32) - 5.0
    for n in range(N):
        mine = lane_experts(E, int(rng.integers(32)))
        lo_n, hi_n = min(3, len(mine)), min(5, len(mine))
        take = rng.permutation(mine)[:int(rng.integers(lo_n, hi_n + 1))]
        x[n, take] = (10.0 - np.arange(len(take))).astype(np.float32)
    return x


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


@pytest.mark.parametrize("E", [64, 96, 128, 160, 192, 224, 256])
@pytest.mark.parametrize("kind", ["normal", "ties", "close", "clustered"])
def test_lane_lists_pass_only_with_the_exact_top_k(E, kind):
    rng = np.random.default_rng(7 * E + len(kind))
    N = 300
    x = clustered(N, E, rng) if kind == "clustered" else rows(kind, N, E, rng)
    idx_or, _ = oracle.gate_topk(x, K)
    idx, passes = lane_list_rule(x)
    assert (idx[passes] == idx_or[passes]).all()
    if kind == "normal":
        assert passes.mean() > 0.9
    elif kind == "clustered":
        # a lane holding three of the leading picks runs out of a three-deep
        # list, or its next key sits below them: with at most three keys a
        # lane, the whole list is kept and the picks stay exact
        if E // 32 > 3:
            assert not passes.any()
        else:
            assert passes.all()
    else:
        assert not passes.any()

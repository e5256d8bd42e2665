"""CPU restatement of the reroute kernel's tile procedure, checked against the
oracle's reroute (CPU only).

The kernel cuts the pairs, in scan order, into tiles of TP pairs and each tile
into 16 sub-ranges, one per warp. A warp counts its sub-range per expert; the
tile publishes its counts, and the exclusive scan over the sub-ranges gives
each sub-range's offset per expert. Each warp then ranks its pairs in rounds
of 32 lanes: a pair's offset in the tile is its sub-range's running count for
its expert plus the lanes of the round below it holding the same expert, and
after the round the count moves on by the round's pairs of that expert. The
look-back gives the tile's exclusive prefix per expert, pre[e], the expert's
pairs in earlier tiles. Per expert the tile keeps one record: the copy that
holds occurrence pre[e], its row for offset 0 and how many offsets stay in
that copy. A pair whose offset is below that bound takes the record; the
others find their copy from their occurrence o = pre[e] + offset: by one
division when the expert's quotas have the floor form b + [j < L mod c], else
as the last copy whose start is at or below o.

The claim pinned here: this procedure gives the oracle's slot and row for
every pair, for the global and the interleaved orders, under the greedy plan,
the capacity planner's arbitrary quotas and plans with zero-quota copies, at
tile sizes from one round per sub-range to the kernel's own, and both the
record and the search are used.

"UltraEP" README, "Interface / 2. Forward and backward" (reroute expands
logical routing to physical replicas); "Performance Tuning / Replication
planning" (the capacity planner, the interleaved order).
"""
import numpy as np
import pytest

import oracle

SUBRANGES = 16
LANES = 32


def copy_table(R, E, S, pl):
    """Per expert, its copies in copy order: (physical slot, first row, quota)."""
    M = E // R
    out = []
    for e in range(E):
        slots = [(e // M) * (M + S) + e % M]
        slots += [(g // S) * (M + S) + M + g % S for g in range(R * S) if pl.slot_expert[g] == e]
        out.append([(p, int(pl.slot_offset[p]), int(pl.slot_quota[p])) for p in slots])
    return out


def copy_holding(cps, L, o):
    """(j, start, end) of the copy holding occurrence o, as the kernel finds it."""
    c = len(cps)
    quotas = [q for _, _, q in cps]
    b, rem = divmod(L, c)
    if all(q == b + (1 if j < rem else 0) for j, q in enumerate(quotas)):
        thr = rem * (b + 1)
        j = o // (b + 1) if o < thr else rem + (o - thr) // b
        start = j * b + min(j, rem)
    else:
        starts = np.concatenate([[0], np.cumsum(quotas)[:-1]])
        j = int(np.nonzero(starts <= o)[0][-1])
        start = int(starts[j])
    return j, start, start + quotas[j]


def scan_order(R, T, K, order):
    if order == "prefix":
        return np.arange(R * T * K)
    return np.array([(r * T + t) * K + k for t in range(T) for r in range(R) for k in range(K)])


def tile_reroute(idx, R, T, E, S, pl, TP, order, used):
    K = idx.shape[1]
    Q = R * T * K
    scan = scan_order(R, T, K, order)
    ids = idx.ravel()[scan]
    cps = copy_table(R, E, S, pl)
    L = np.bincount(ids, minlength=E)
    phys = np.full(Q, -1, dtype=np.int64)
    dest = np.full(Q, -1, dtype=np.int64)
    pre = np.zeros(E, dtype=np.int64)  # what the look-back returns, tile by tile
    sub = TP // SUBRANGES
    for t0 in range(0, Q, TP):
        tile = ids[t0:t0 + TP]
        # counts per sub-range, then each sub-range's offset per expert
        counts = np.zeros((SUBRANGES, E), dtype=np.int64)
        for w in range(SUBRANGES):
            seg = tile[w * sub:(w + 1) * sub]
            counts[w] = np.bincount(seg, minlength=E)
        run = np.cumsum(counts, axis=0) - counts
        # ranks, round by round within each sub-range
        offset = np.empty(len(tile), dtype=np.int64)
        for w in range(SUBRANGES):
            for r0 in range(w * sub, min((w + 1) * sub, len(tile)), LANES):
                rnd = tile[r0:min(r0 + LANES, (w + 1) * sub, len(tile))]
                for lane, e in enumerate(rnd):
                    offset[r0 + lane] = run[w, e] + int(np.sum(rnd[:lane] == e))
                for e in np.unique(rnd):
                    run[w, e] += int(np.sum(rnd == e))
        # the record of each expert's first pair in the tile
        rec = {}
        for e in np.unique(tile):
            if pre[e] < L[e]:
                j, start, end = copy_holding(cps[e], int(L[e]), int(pre[e]))
                p, row0, _ = cps[e][j]
                rec[e] = (p, row0 + int(pre[e]) - start, end - int(pre[e]))
        for x, e in enumerate(tile):
            lo = int(offset[x])
            if e in rec and lo < rec[e][2]:
                p, row = rec[e][0], rec[e][1] + lo
                used["record"] += 1
            else:
                o = int(pre[e]) + lo
                j, start, _ = copy_holding(cps[e], int(L[e]), o)
                p, row = cps[e][j][0], cps[e][j][1] + o - start
                used["search"] += 1
            phys[scan[t0 + x]] = p
            dest[scan[t0 + x]] = row
        pre += np.bincount(tile, minlength=E)
    return phys.reshape(idx.shape), dest.reshape(idx.shape)


def skewed_logits(R, T, E, seed, boost=(3.0, 1.5)):
    rng = np.random.default_rng(seed)
    lg = rng.normal(size=(R * T, E)).astype(np.float32)
    lg[:, 0] += boost[0]
    lg[:, 1] += boost[1]
    return lg


CASES = [
    # R, T, E, K, S, planner, seed
    (8, 48, 64, 4, 2, "greedy", 1),
    (8, 48, 64, 4, 2, "bisect", 1),
    (4, 40, 16, 3, 2, "bisect", 2),
    (4, 1, 8, 1, 4, "greedy", 3),   # copies outnumber pairs: zero quotas
    (3, 1, 6, 1, 2, "greedy", 0),
    (5, 12, 20, 2, 3, "greedy", 4),
]


@pytest.fixture(scope="module")
def usage():
    used = {"record": 0, "search": 0}
    yield used
    assert used["record"] > 0 and used["search"] > 0


@pytest.mark.parametrize("R,T,E,K,S,planner,seed", CASES)
@pytest.mark.parametrize("TP", [SUBRANGES * LANES, SUBRANGES * LANES * 3, 512 * 7])
@pytest.mark.parametrize("order", ["prefix", "interleave"])
def test_tile_procedure_matches_the_oracle(R, T, E, K, S, planner, seed, TP, order, usage):
    lg = skewed_logits(R, T, E, seed)
    idx, _ = oracle.gate_topk(lg, K)
    _, load_e = oracle.count(idx, R, T, E)
    if planner == "greedy":
        pl = oracle.plan(load_e, R, S)
    else:
        pl = oracle.plan_bisect(load_e, R, S, min_tokens=2)
    if order == "prefix":
        phys_or, dest_or = oracle.reroute(idx, R, E, S, pl)
    else:
        phys_or, dest_or = oracle.reroute_interleave(idx, R, T, E, S, pl)
    phys, dest = tile_reroute(idx, R, T, E, S, pl, TP, order, usage)
    np.testing.assert_array_equal(phys, phys_or)
    np.testing.assert_array_equal(dest, dest_or)

"""Pins for the oracle's replication plan and reroute (CPU only).

* Hand-worked plans (tests/golden/plan_cases.json) fix every rule: tie
  breaks, remainder order, stop test, forced placements.
* Invariants that any correct plan satisfies, on random skewed loads.
* An exhaustive search over every filling of the redundant slots bounds the
  greedy makespan from below: ceil(Q/R) <= OPT <= greedy.
* The reroute is pinned by a hand-worked example and by invariants that
  determine it completely given the plan (prefix fill in global order).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle


def load_cases(golden_dir):
    with open(os.path.join(golden_dir, "plan_cases.json")) as f:
        return json.load(f)["cases"]


def test_hand_worked_plans(golden_dir):
    for c in load_cases(golden_dir):
        pl = oracle.plan(np.array(c["load_e"], dtype=np.int32), c["R"], c["S"])
        got = dict(slot_expert=pl.slot_expert.tolist(),
                   n_copies=pl.n_copies.tolist(),
                   slot_quota=pl.slot_quota.tolist(),
                   slot_offset=pl.slot_offset.tolist(),
                   rank_load=pl.rank_load.tolist(),
                   stats=pl.stats.tolist(),
                   trace_e=pl.trace_e.tolist(), trace_r=pl.trace_r.tolist())
        for key, val in got.items():
            assert val == c[key], (c["name"], key, val, c[key])


def copies_of(pl, E, R, S):
    """Physical slots of every expert's copies, in copy order."""
    M = E // R
    out = []
    for e in range(E):
        lst = [(e // M) * (M + S) + e % M]
        for g in range(R * S):
            if pl.slot_expert[g] == e:
                lst.append((g // S) * (M + S) + M + g % S)
        out.append(lst)
    return out


def check_plan_invariants(load_e, R, S, pl):
    E = len(load_e)
    M = E // R
    G = R * S
    Q = int(np.sum(load_e))
    cps = copies_of(pl, E, R, S)
    for e in range(E):
        q = [int(pl.slot_quota[p]) for p in cps[e]]
        assert sum(q) == load_e[e]
        assert max(q) - min(q) <= 1
        assert all(q[j] >= q[j + 1] for j in range(len(q) - 1))
        assert pl.n_copies[e] == len(cps[e])
    empty = [g for g in range(G) if pl.slot_expert[g] < 0]
    for g in empty:
        assert pl.slot_quota[(g // S) * (M + S) + M + g % S] == 0
    # slots on a rank fill from the lowest index: no holes
    for r in range(R):
        used = [pl.slot_expert[r * S + s] >= 0 for s in range(S)]
        assert used == sorted(used, reverse=True)
    np.testing.assert_array_equal(pl.slot_offset,
                                  np.concatenate([[0], np.cumsum(pl.slot_quota)]))
    per_rank = pl.slot_quota.reshape(R, M + S).sum(axis=1)
    np.testing.assert_array_equal(pl.rank_load, per_rank)
    assert pl.rank_load.sum() == Q
    mx = int(pl.rank_load.max())
    assert pl.stats[2] == mx
    assert mx >= math.ceil(Q / R)
    assert 50 * R * mx <= 51 * Q or len(empty) == 0
    assert pl.stats[0] == G - len(empty) == len(pl.trace_e)
    assert pl.stats[1] == int(np.asarray(load_e).reshape(R, M).sum(axis=1).max())


def zipf_loads(rng, E, K, N, s):
    w = (np.arange(1, E + 1, dtype=np.float64)) ** (-s)
    w = w[rng.permutation(E)]
    w /= w.sum()
    return rng.multinomial(N * K, w).astype(np.int32)


@pytest.mark.parametrize("R,E,S,s", [(8, 64, 2, 1.2), (64, 128, 2, 1.0), (64, 256, 2, 1.3),
                                     (40, 160, 1, 1.1), (4, 4, 3, 2.0), (3, 9, 1, 0.5),
                                     (16, 16, 8, 1.5)])
def test_plan_invariants_random(R, E, S, s):
    rng = np.random.default_rng(R * 1000 + E + S)
    for _ in range(5):
        load_e = zipf_loads(rng, E, 8, 512 * R, s)
        pl = oracle.plan(load_e, R, S)
        check_plan_invariants(load_e, R, S, pl)


def test_plan_uniform_exact_no_copies():
    for R, E, S in [(8, 64, 2), (64, 128, 2), (64, 256, 2), (40, 160, 1)]:
        load_e = np.full(E, 4096, dtype=np.int32)
        pl = oracle.plan(load_e, R, S)
        assert pl.stats[0] == 0
        assert (pl.slot_expert == -1).all()
        assert (pl.n_copies == 1).all()


def test_plan_single_hot_expert_closed_form():
    # all 800 pairs on expert 5 (master on rank 2), R=4, S=2: the greedy adds
    # one copy on each other rank, lowest rank first (r0, r1, r3); with 4
    # copies every rank carries 200 = mean, so it stops with slots left
    R, E, S = 4, 8, 2
    load_e = np.zeros(E, dtype=np.int32)
    load_e[5] = 800
    pl = oracle.plan(load_e, R, S)
    assert pl.slot_expert.tolist() == [5, -1, 5, -1, -1, -1, 5, -1]
    assert pl.trace_r.tolist() == [0, 1, 3]
    assert pl.rank_load.tolist() == [200, 200, 200, 200]
    assert pl.stats.tolist() == [3, 800, 200, 0]


def brute_opt(load_e, R, S):
    """Smallest makespan over every filling of the G redundant slots, with
    the same quota rule (ascending slot order for the remainders)."""
    E = len(load_e)
    M = E // R
    G = R * S
    best = None
    for fill in itertools.product(range(-1, E), repeat=G):
        loads = [0] * R
        for e in range(E):
            L = int(load_e[e])
            reps = [g for g in range(G) if fill[g] == e]
            c = 1 + len(reps)
            ranks = [e // M] + [g // S for g in reps]
            for j, r in enumerate(ranks):
                loads[r] += L // c + (1 if j < L % c else 0)
        m = max(loads)
        best = m if best is None else min(best, m)
    return best


@pytest.mark.parametrize("R,E,S", [(2, 4, 1), (2, 2, 2), (3, 6, 1), (2, 6, 2), (4, 4, 1)])
def test_plan_bounded_by_exhaustive_opt(R, E, S):
    rng = np.random.default_rng(R * 31 + E * 7 + S)
    ratios = []
    for _ in range(6):
        load_e = zipf_loads(rng, E, 2, 20 * R, 1.5)
        Q = int(load_e.sum())
        pl = oracle.plan(load_e, R, S)
        opt = brute_opt(load_e, R, S)
        greedy = int(pl.rank_load.max())
        assert math.ceil(Q / R) <= opt <= greedy
        ratios.append(greedy / opt)
    # the pages state no approximation bound; a large ratio is a finding only
    assert max(ratios) < 3.0


def test_reroute_hand_worked(golden_dir):
    with open(os.path.join(golden_dir, "reroute_case.json")) as f:
        c = json.load(f)
    idx = np.array(c["idx"], dtype=np.int32)
    load_re, load_e = oracle.count(idx, c["R"], c["T"], c["E"])
    pl = oracle.plan(load_e, c["R"], c["S"])
    phys, dest = oracle.reroute(idx, c["R"], c["E"], c["S"], pl)
    assert phys.tolist() == c["phys_slot"]
    assert dest.tolist() == c["dest_row"]


def check_reroute_determined(idx, R, E, S, pl, phys, dest):
    """Given the plan, these properties leave exactly one valid result:
    every pair goes to a copy of its own expert; each expert's pairs, in
    global order, fill its copies' row ranges one after another in copy
    order."""
    M = E // R
    Q = idx.size
    flat_e = idx.ravel()
    flat_p = phys.ravel()
    flat_d = dest.ravel().astype(np.int64)
    slot_owner = np.empty(R * (M + S), dtype=np.int64)
    for p in range(R * (M + S)):
        r, l = divmod(p, M + S)
        slot_owner[p] = r * M + l if l < M else pl.slot_expert[r * S + l - M]
    assert (slot_owner[flat_p] == flat_e).all()
    assert np.array_equal(np.sort(flat_d), np.arange(Q))
    cps = copies_of(pl, E, R, S)
    order = np.argsort(flat_e, kind="stable")  # pairs grouped by expert, global order kept
    starts = np.concatenate([[0], np.cumsum(np.bincount(flat_e, minlength=E))])
    for e in range(E):
        pairs = order[starts[e]:starts[e + 1]]
        expect_rows = np.concatenate(
            [np.arange(pl.slot_offset[p], pl.slot_offset[p] + pl.slot_quota[p]) for p in cps[e]]
            + [np.zeros(0, dtype=np.int64)])
        expect_slots = np.concatenate(
            [np.full(pl.slot_quota[p], p) for p in cps[e]] + [np.zeros(0, dtype=np.int64)])
        np.testing.assert_array_equal(flat_d[pairs], expect_rows)
        np.testing.assert_array_equal(flat_p[pairs], expect_slots)


@pytest.mark.parametrize("R,T,E,K,S", [(8, 64, 64, 4, 2), (4, 33, 16, 3, 2), (3, 50, 9, 2, 1),
                                       (2, 40, 4, 4, 3), (5, 20, 10, 1, 0)])
def test_reroute_invariants_random(R, T, E, K, S):
    rng = np.random.default_rng(R + T + E + K + S)
    bias = np.log(np.arange(1, E + 1)) * -1.5
    logits = (rng.standard_normal((R * T, E)) + bias[rng.permutation(E)]).astype(np.float32)
    out = oracle.run_path(logits, R, T, S, K)
    check_plan_invariants(out["load_e"], R, S, out["plan"])
    check_reroute_determined(out["idx"], R, E, S, out["plan"], out["phys_slot"],
                             out["dest_row"])


def test_plan_that_cannot_balance_places_zero_quota_copies():
    """Worked by hand: R = 2, E = 2 (one master per rank), S = 3, loads
    L = (3, 0). Q = 3 over 2 ranks can never reach max <= 1.02 * 1.5, so the
    greedy places a copy of expert 0 (the only ratio above 0) in every slot:
    r* = 1, 1, 0, 1, 0, 0 (rank loads (3,0) (2,1) (1,2) (2,1) (2,1) (3,0)).
    With c copies in copy order (master, then ascending g) the quotas are
    floor(3/c) + [j < 3 mod c]: from c = 4 on, every copy past the third
    gets 0, and the last placements move rank 1's pair back to rank 0, so
    the makespan ends where it began. Co-located copies: three on rank 0
    (beside the master) and two on rank 1 (after its first copy)."""
    pl = oracle.plan(np.array([3, 0], dtype=np.int32), 2, 3)
    assert pl.slot_expert.tolist() == [0, 0, 0, 0, 0, 0]
    assert pl.n_copies.tolist() == [7, 1]
    assert pl.slot_quota.tolist() == [1, 1, 1, 0, 0, 0, 0, 0]
    assert pl.slot_offset.tolist() == [0, 1, 2, 3, 3, 3, 3, 3, 3]
    assert pl.rank_load.tolist() == [3, 0]
    assert pl.stats.tolist() == [6, 3, 3, 5]


@pytest.mark.parametrize("R,E,S,seed", [(3, 6, 2, 0), (4, 8, 4, 3), (5, 10, 3, 0)])
def test_reroute_with_zero_quota_copies(R, E, S, seed):
    """Layouts the greedy cannot balance (the hot expert's master shares its
    rank with a master that keeps the remainder), one token per rank, K = 1:
    experts end with more copies than pairs; the reroute still fills the
    copies with a positive quota in copy order and sends nothing to the
    others."""
    rng = np.random.default_rng(seed)
    logits = rng.normal(size=(R, E)).astype(np.float32)
    logits[:, 0] += 4.0
    logits[:, 1] += 2.0
    out = oracle.run_path(logits, R, 1, S, 1)
    pl = out["plan"]
    L = out["load_e"]
    assert ((pl.n_copies > L) & (L > 0)).any()
    check_plan_invariants(L, R, S, pl)
    check_reroute_determined(out["idx"], R, E, S, pl, out["phys_slot"], out["dest_row"])
    used = np.bincount(out["phys_slot"].ravel(), minlength=R * (E // R + S))
    assert (used[pl.slot_quota == 0] == 0).all()

"""Pins for the oracle's planner variants (CPU only).

The UltraEP README ("Performance Tuning / Replication planning") names the
knobs of its own planner: a balancing binary search with an early-stop
target and a ratio tolerance eps, a quota oracle, a minimal load per replica,
zero-load masters, a locality-aware per-rank quota decomposition and an
interleaved reroute order. The pages give no algorithm for them; the oracle
states the project's reading, and these tests pin it:

* hand-worked cases (tests/golden/variant_cases.json) fix every rule:
  shedding order, demand order, receiver choice and ties, the cut and raise
  rules of the minimum, every step of the bisection, the zero-master switch,
  the greedy's minimum, both passes of the locality split;
* invariants that any plan of these rules satisfies, on random skewed loads;
* the bisection's own invariant, through the early-stop path: the grid point
  just below the result is infeasible;
* an exhaustive search over tiny placements bounds the capacity plan's
  makespan from below (Hall's condition for divisible loads);
* the locality split never sends more pairs off their rank than the plain
  prefix fill, and its reroute is fully determined by the split;
* the interleaved reroute equals the plain reroute run on the pairs taken in
  (token, rank, k) order.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from tests.test_oracle_plan import check_reroute_determined, copies_of, zipf_loads


def cases(golden_dir, kind):
    with open(os.path.join(golden_dir, "variant_cases.json")) as f:
        return json.load(f)[kind]


def plan_dict(pl):
    return dict(slot_expert=pl.slot_expert.tolist(), n_copies=pl.n_copies.tolist(),
                slot_quota=pl.slot_quota.tolist(), slot_offset=pl.slot_offset.tolist(),
                rank_load=pl.rank_load.tolist(), stats=pl.stats.tolist())


# ---------------------------------------------------------------- hand cases

def test_bisect_hand_cases(golden_dir):
    for c in cases(golden_dir, "bisect"):
        pl = oracle.plan_bisect(np.array(c["load_e"], dtype=np.int32), c["R"], c["S"],
                                eps_inv=c["eps_inv"], threshold=c["threshold"],
                                min_tokens=c["min_tokens"],
                                allow_zero_master=bool(c["allow_zero"]))
        for key, val in plan_dict(pl).items():
            assert val == c[key], (c["name"], key, val, c[key])


def test_greedy_min_tokens_hand_cases(golden_dir):
    for c in cases(golden_dir, "greedy_min_tokens"):
        pl = oracle.plan(np.array(c["load_e"], dtype=np.int32), c["R"], c["S"],
                         min_tokens=c["min_tokens"])
        got = plan_dict(pl)
        got.update(trace_e=pl.trace_e.tolist(), trace_r=pl.trace_r.tolist())
        for key, val in got.items():
            assert val == c[key], (c["name"], key, val, c[key])


def test_locality_split_hand_cases(golden_dir):
    for c in cases(golden_dir, "locality_split"):
        pl = oracle.Plan(np.array(c["slot_expert"], dtype=np.int32), None,
                         np.array(c["slot_quota"], dtype=np.int32),
                         np.array(c["slot_offset"], dtype=np.int32), None, None, None, None)
        sq, so = oracle.locality_split(np.array(c["load_re"], dtype=np.int32), c["S"], pl)
        assert sq.tolist() == c["src_quota"], c["name"]
        assert so.tolist() == c["src_offset"], c["name"]


# ------------------------------------------------------- capacity planner

def capacity(k, Q, D, R):
    return k * Q // (D * R)


def check_bisect_invariants(load_e, R, S, pl, D, thr, m, allow_zero):
    E = len(load_e)
    M = E // R
    G = R * S
    Q = int(np.sum(load_e))
    H = np.asarray(load_e, dtype=np.int64).reshape(R, M).sum(axis=1)
    probes, max_before, max_after, k = (int(v) for v in pl.stats)
    assert max_before == int(H.max())
    C = capacity(k, Q, D, R)
    cps = copies_of(pl, E, R, S)
    for e in range(E):
        q = [int(pl.slot_quota[p]) for p in cps[e]]
        assert sum(q) == load_e[e], e
        assert all(x >= m for x in q[1:]), (e, q)           # every replica >= m
        if not allow_zero and load_e[e] > 0:
            assert q[0] >= 1, e                             # master keeps a pair
        hosts = [p // (M + S) for p in cps[e][1:]]
        assert e // M not in hosts                          # never on the master rank
        assert len(set(hosts)) == len(hosts)                # one replica per rank
        assert pl.n_copies[e] == len(cps[e])
        if len(q) > 1:                                      # only overflow ranks shed
            assert H[e // M] > C
    for r in range(R):
        used = [pl.slot_expert[r * S + s] >= 0 for s in range(S)]
        assert used == sorted(used, reverse=True)           # lowest free slot first
    for g in range(G):
        if pl.slot_expert[g] < 0:
            assert pl.slot_quota[(g // S) * (M + S) + M + g % S] == 0
    np.testing.assert_array_equal(pl.slot_offset,
                                  np.concatenate([[0], np.cumsum(pl.slot_quota)]))
    np.testing.assert_array_equal(pl.rank_load, pl.slot_quota.reshape(R, M + S).sum(axis=1))
    assert pl.rank_load.sum() == Q
    assert max_after == int(pl.rank_load.max()) <= max(C, 0) or (Q == 0 and max_after == 0)
    assert k >= thr
    if k > thr:
        # the bisection ends with lo = k - 1 probed infeasible: asking the
        # planner to start there must not stop early at k - 1
        below = oracle.plan_bisect(load_e, R, S, eps_inv=D, threshold=k - 1, min_tokens=m,
                                   allow_zero_master=allow_zero)
        assert int(below.stats[3]) != k - 1
        # and k itself is the grid point where C first reaches max H, or a
        # point the search probed; either way C(k) <= C(hi_start)
        assert C <= max(int(H.max()), capacity(math.ceil(D * R * int(H.max()) / Q), Q, D, R))
        assert probes >= 2
    else:
        assert probes == 1


@pytest.mark.parametrize("R,E,S,s,m", [(8, 64, 2, 1.2, 16), (64, 128, 2, 1.0, 1024),
                                       (64, 256, 2, 1.3, 1024), (40, 160, 1, 1.1, 1024),
                                       (4, 4, 3, 2.0, 1), (3, 9, 1, 0.5, 8), (16, 16, 8, 1.5, 64)])
def test_bisect_invariants_random(R, E, S, s, m):
    rng = np.random.default_rng(R * 1000 + E + S + m)
    for trial in range(4):
        load_e = zipf_loads(rng, E, 8, 512 * R, s)
        for D, allow_zero in ((100, False), (1000, True)):
            pl = oracle.plan_bisect(load_e, R, S, eps_inv=D, min_tokens=m,
                                    allow_zero_master=allow_zero)
            check_bisect_invariants(load_e, R, S, pl, D, D, m, allow_zero)


def test_bisect_uniform_and_empty():
    for R, E, S in [(8, 64, 2), (64, 128, 2), (40, 160, 1)]:
        pl = oracle.plan_bisect(np.full(E, 4096, dtype=np.int32), R, S)
        assert pl.stats.tolist()[0] == 1 and pl.stats[3] == 100   # feasible at 1.0
        assert (pl.slot_expert == -1).all()
        pl = oracle.plan_bisect(np.zeros(E, dtype=np.int32), R, S)
        assert (pl.slot_expert == -1).all() and pl.rank_load.sum() == 0


def test_bisect_threshold_above_start_stops_at_once():
    # threshold 3.0 on a 2.5x skew: C(300) covers max H, no replica, 1 probe
    load_e = np.array([250, 50, 50, 50], dtype=np.int32)     # H = [250, 50, 50, 50], mean 100
    pl = oracle.plan_bisect(load_e, 4, 1, threshold=300, min_tokens=1)
    assert pl.stats.tolist() == [1, 250, 250, 300]
    assert (pl.slot_expert == -1).all()


def hall_opt(load_e, R, S):
    """Smallest integer makespan over every filling of the redundant slots,
    each expert's load split freely over the ranks holding its copies: for a
    fixed filling, max over expert sets U of ceil(L(U) / |ranks of U|)."""
    E = len(load_e)
    M = E // R
    G = R * S
    best = None
    for fill in itertools.product(range(-1, E), repeat=G):
        hosts = [{e // M} for e in range(E)]
        for g, e in enumerate(fill):
            if e >= 0:
                hosts[e].add(g // S)
        worst = 0
        for mask in range(1, 1 << E):
            U = [e for e in range(E) if mask >> e & 1]
            load = sum(int(load_e[e]) for e in U)
            ranks = set().union(*(hosts[e] for e in U))
            worst = max(worst, -(-load // len(ranks)))
        best = worst if best is None else min(best, worst)
    return best


@pytest.mark.parametrize("R,E,S", [(2, 4, 1), (2, 2, 2), (3, 3, 1), (2, 4, 2)])
def test_bisect_bounded_by_exhaustive_opt(R, E, S):
    rng = np.random.default_rng(R * 17 + E * 5 + S)
    for _ in range(5):
        load_e = zipf_loads(rng, E, 2, 30 * R, 1.5)
        Q = int(load_e.sum())
        pl = oracle.plan_bisect(load_e, R, S, min_tokens=1)
        opt = hall_opt(load_e, R, S)
        assert math.ceil(Q / R) <= opt <= int(pl.rank_load.max())


def test_bisect_reroute_fills_general_quotas():
    # the plain reroute, given a capacity plan (quotas not of the floor form),
    # is still the prefix fill its invariants determine
    rng = np.random.default_rng(5)
    R, T, E, K, S = 4, 50, 8, 3, 2
    idx = np.stack([rng.choice(E, K, replace=False, p=np.r_[0.4, np.full(7, 0.6 / 7)])
                    for _ in range(R * T)]).astype(np.int32)
    _, load_e = oracle.count(idx, R, T, E)
    pl = oracle.plan_bisect(load_e, R, S, min_tokens=4)
    assert (pl.slot_expert >= 0).any()
    phys, dest = oracle.reroute(idx, R, E, S, pl)
    check_reroute_determined(idx, R, E, S, pl, phys, dest)


# ------------------------------------------------- greedy with a minimum

@pytest.mark.parametrize("R,E,S,s,m", [(8, 64, 2, 1.2, 64), (64, 128, 2, 1.0, 1024),
                                       (40, 160, 1, 1.1, 4096), (4, 4, 3, 2.0, 100)])
def test_greedy_min_tokens_invariants(R, E, S, s, m):
    rng = np.random.default_rng(R + E + S + m)
    for _ in range(4):
        load_e = zipf_loads(rng, E, 8, 512 * R, s)
        Q = int(load_e.sum())
        pl = oracle.plan(load_e, R, S, min_tokens=m)
        cps = copies_of(pl, E, R, S)
        for e in range(E):
            q = [int(pl.slot_quota[p]) for p in cps[e]]
            assert sum(q) == load_e[e] and max(q) - min(q) <= 1
            if len(q) > 1:
                assert min(q) >= m                      # every copy keeps >= m
        free = int((pl.slot_expert < 0).sum())
        mx = int(pl.rank_load.max())
        if free and 50 * R * mx > 51 * Q:
            # stopped early: no expert may take another copy
            assert all(load_e[e] < m * (pl.n_copies[e] + 1) for e in range(E))
    # m = 0 is the plain greedy
    load_e = zipf_loads(rng, E, 8, 512 * R, s)
    a, b = oracle.plan(load_e, R, S), oracle.plan(load_e, R, S, min_tokens=0)
    assert plan_dict(a) == plan_dict(b)


# ------------------------------------------------------- locality split

def remote_pairs(src_quota, R, M, S):
    P = src_quota.shape[1]
    host = np.arange(P) // (M + S)
    return int(sum(src_quota[r, host != r].sum() for r in range(R)))


def prefix_src_quota(idx, R, T, E, S, pl):
    """Pairs per (source rank, slot) under the plain prefix-fill reroute."""
    M = E // R
    phys, _ = oracle.reroute(idx, R, E, S, pl)
    P = R * (M + S)
    src = np.arange(idx.size) // (T * idx.shape[1])
    out = np.zeros((R, P), dtype=np.int64)
    np.add.at(out, (src, phys.ravel()), 1)
    return out


def skewed_routing(rng, R, T, E, K, s, per_rank_perm=False):
    """Top-K ids per token from Zipf-biased logits (optionally a different hot
    set per source rank)."""
    idx = np.empty((R * T, K), dtype=np.int32)
    w0 = (np.arange(1, E + 1, dtype=np.float64)) ** (-s)
    for r in range(R):
        w = w0[rng.permutation(E)] if (per_rank_perm or r == 0) else w
        g = rng.gumbel(size=(T, E)) + np.log(w)
        idx[r * T:(r + 1) * T] = np.argsort(-g, axis=1, kind="stable")[:, :K]
    return idx


@pytest.mark.parametrize("R,T,E,K,S,per_rank", [(4, 64, 8, 2, 2, False), (8, 128, 64, 4, 2, True),
                                                (3, 37, 6, 3, 2, True), (16, 64, 32, 8, 1, False)])
@pytest.mark.parametrize("planner", ["greedy", "bisect"])
def test_locality_split_invariants(R, T, E, K, S, per_rank, planner):
    rng = np.random.default_rng(R * T + E + K + S)
    M = E // R
    idx = skewed_routing(rng, R, T, E, K, 1.2, per_rank)
    load_re, load_e = oracle.count(idx, R, T, E)
    pl = (oracle.plan(load_e, R, S) if planner == "greedy"
          else oracle.plan_bisect(load_e, R, S, min_tokens=4))
    sq, so = oracle.locality_split(load_re, S, pl)
    cps = copies_of(pl, E, R, S)
    np.testing.assert_array_equal(sq.sum(axis=0), pl.slot_quota)    # columns: quotas
    for e in range(E):
        np.testing.assert_array_equal(sq[:, cps[e]].sum(axis=1), load_re[:, e])
        # local first: a copy alone on its host takes min(host's pairs, quota)
        hosts = [p // (M + S) for p in cps[e]]
        for p, h in zip(cps[e], hosts):
            if hosts.count(h) == 1:
                assert sq[h, p] == min(load_re[h, e], pl.slot_quota[p])
    for p in range(sq.shape[1]):
        np.testing.assert_array_equal(
            so[:, p], pl.slot_offset[p] + np.concatenate([[0], np.cumsum(sq[:-1, p])]))
    assert remote_pairs(sq, R, M, S) <= remote_pairs(prefix_src_quota(idx, R, T, E, S, pl), R, M, S)
    # the reroute under the split
    phys, dest = oracle.reroute_local(idx, R, T, E, S, pl, sq, so)
    check_local_reroute(idx, R, T, E, S, pl, sq, so, phys, dest)


def check_local_reroute(idx, R, T, E, S, pl, sq, so, phys, dest):
    """Given the split, one result is valid: source rank r hands its pairs of
    e, in its own order, to e's copies in copy order, sq[r][p] each, at rows
    so[r][p], so[r][p] + 1, ..."""
    M = E // R
    K = idx.shape[1]
    cps = copies_of(pl, E, R, S)
    assert np.array_equal(np.sort(dest.ravel()), np.arange(idx.size))
    for r in range(R):
        blk = slice(r * T * K, (r + 1) * T * K)
        e_r, p_r, d_r = idx.ravel()[blk], phys.ravel()[blk], dest.ravel()[blk]
        for e in range(E):
            sel = np.nonzero(e_r == e)[0]
            want_p = np.concatenate([np.full(sq[r, p], p) for p in cps[e]] + [np.zeros(0, int)])
            want_d = np.concatenate([so[r, p] + np.arange(sq[r, p]) for p in cps[e]]
                                    + [np.zeros(0, int)])
            np.testing.assert_array_equal(p_r[sel], want_p)
            np.testing.assert_array_equal(d_r[sel], want_d)


def prefix_src_quota_from_loads(load_re, pl, R, S):
    """Pairs per (source rank, slot) under the plain prefix fill, from the
    loads alone: in global order expert e's pairs from source r occupy
    positions [pre_r, pre_r + s_r), copy j takes [start_j, start_j + q_j)."""
    E = load_re.shape[1]
    P = pl.slot_quota.size
    out = np.zeros((R, P), dtype=np.int64)
    for e, cp in enumerate(copies_of(pl, E, R, S)):
        pre = np.concatenate([[0], np.cumsum(load_re[:, e])])
        start = 0
        for p in cp:
            q = int(pl.slot_quota[p])
            for r in range(R):
                lo, hi = max(pre[r], start), min(pre[r + 1], start + q)
                out[r, p] += max(0, hi - lo)
            start += q
    return out


def test_locality_cuts_remote_pairs_of_a_hot_expert(golden_dir):
    # the hand case: prefix fill sends 280 pairs off their rank (expert 1:
    # rank 0's 150 to the master on rank 1, rank 1's last 100 to the replica
    # on rank 0; expert 0: rank 1's 30), the split 80
    c = cases(golden_dir, "locality_split")[0]
    load_re = np.array(c["load_re"], dtype=np.int32)
    pl = oracle.Plan(np.array(c["slot_expert"], dtype=np.int32), None,
                     np.array(c["slot_quota"], dtype=np.int32),
                     np.array(c["slot_offset"], dtype=np.int32), None, None, None, None)
    sq, so = oracle.locality_split(load_re, 1, pl)
    assert remote_pairs(sq, 2, 1, 1) == 80
    assert remote_pairs(prefix_src_quota_from_loads(load_re, pl, 2, 1), 2, 1, 1) == 280


# ------------------------------------------------------ interleaved order

@pytest.mark.parametrize("R,T,E,K,S", [(4, 64, 8, 2, 2), (8, 128, 64, 4, 2), (3, 37, 6, 3, 2),
                                       (16, 16, 32, 8, 1), (1, 20, 4, 2, 1)])
@pytest.mark.parametrize("planner", ["greedy", "bisect"])
def test_interleave_is_prefix_fill_in_token_major_order(R, T, E, K, S, planner):
    rng = np.random.default_rng(R + T + E)
    idx = skewed_routing(rng, R, T, E, K, 1.4, True)
    _, load_e = oracle.count(idx, R, T, E)
    pl = (oracle.plan(load_e, R, S) if planner == "greedy"
          else oracle.plan_bisect(load_e, R, S, min_tokens=2))
    phys, dest = oracle.reroute_interleave(idx, R, T, E, S, pl)
    # the same pairs taken in (t, r, k) order through the plain reroute
    perm = idx.reshape(R, T, K).transpose(1, 0, 2).reshape(R * T, K)
    p2, d2 = oracle.reroute(np.ascontiguousarray(perm), R, E, S, pl)
    back = lambda a: a.reshape(T, R, K).transpose(1, 0, 2).reshape(R * T, K)
    np.testing.assert_array_equal(phys, back(p2))
    np.testing.assert_array_equal(dest, back(d2))
    # and that result is the one the fill invariants determine
    check_reroute_determined(np.ascontiguousarray(perm), R, E, S, pl, p2, d2)
    if R > 1 and planner == "greedy" and (pl.slot_expert >= 0).any():
        # a replicated expert's copies now draw pairs from every source rank
        e = int(pl.slot_expert[pl.slot_expert >= 0][0])
        M = E // R
        master = (e // M) * (M + S) + e % M
        src = np.nonzero((idx == e).any(axis=1))[0] // T
        from_master = np.unique(src[(phys == master)[(idx == e).any(axis=1)].any(axis=1)])
        assert from_master.size > 1 or np.unique(src).size == 1

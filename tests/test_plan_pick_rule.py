"""CPU check of the decomposition behind the plan kernel (CPU only).

The greedy chooses e* = argmax L_e/c_e (ties to the lowest e) at every step,
and the choice depends only on the copy counts, never on the ranks. Each
expert's successive ratios L/1, L/2, ... fall, so the greedy's picks are the
merge of those lists: the keys (L_e/c, e), c = 1, 2, ..., in descending ratio
(equal ratios: lower e first), each list cut where the expert may not grow
(with a minimum of m pairs per replica, copy c+1 needs L >= m (c+1)). The
kernel computes that pick sequence in parallel, as keys
floor(L 2^17 / c) * 2^16 + (255 - e) * 2^8 + (c - 1), exact for c <= 257,
and then runs only the rank side serially: stop when 50 R max load <= 51 Q
(in the kernel: max load <= floor(51 Q / (50 R))) or no slot is free or the
picks run out; else the least loaded rank with a free slot (ties to the
lowest r) takes the next pick in its lowest free slot, and the expert's
copies get the quotas floor(L/c) + [j < L mod c] in copy order (master, then
ascending slot).

That procedure is restated below and checked against the oracle's greedy,
which recomputes every ratio and load from scratch at each step, on random
skewed loads, with and without a minimum per replica, and on layouts where
copies outnumber pairs.

"How balancing in 300 microseconds works" (quota-driven scheduler); "UltraEP"
README, "Interface / 2. Forward and backward" (update_placement),
"Performance Tuning / Replication planning" (minimal load per replica).
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle


def pick_sequence(load_e, G, min_tokens):
    """The greedy's expert picks, in order, from the loads alone: the kernel's
    integer keys, checked against exact fractions."""
    keys = []
    for e, L in enumerate(int(x) for x in load_e):
        if L <= 0:
            continue
        cap = G if min_tokens == 0 else min(G, L // min_tokens - 1)
        for c in range(1, cap + 1):
            keys.append(((L << 17) // c, 255 - e, c - 1, Fraction(L, c), e))
    keys.sort(key=lambda k: (k[0], k[1], k[2]), reverse=True)
    exact = sorted(keys, key=lambda k: (k[3], -k[4]), reverse=True)
    assert [k[4] for k in keys] == [k[4] for k in exact]
    return [k[4] for k in keys[:G]]


def plan_by_picks(load_e, R, S, min_tokens=0):
    E = len(load_e)
    M = E // R
    G = R * S
    Q = int(np.sum(load_e))
    picks = pick_sequence(load_e, G, min_tokens)
    copies = [1] * E
    slot_expert = [-1] * G
    used = [0] * R

    def rank_loads():
        load = [0] * R
        for e in range(E):
            L, c = int(load_e[e]), copies[e]
            slots = [(e // M)] + [g // S for g in range(G) if slot_expert[g] == e]
            for j, r in enumerate(slots):
                load[r] += L // c + (1 if j < L % c else 0)
        return load

    load = rank_loads()
    max_before = max(load) if R else 0
    stop_max = (51 * Q) // (50 * R)
    iters = 0
    for e in picks:
        if max(load) <= stop_max:
            break
        free = [r for r in range(R) if used[r] < S]
        if not free:
            break
        rstar = min(free, key=lambda r: (load[r], r))
        slot_expert[rstar * S + used[rstar]] = e
        used[rstar] += 1
        copies[e] += 1
        iters += 1
        load = rank_loads()
    return slot_expert, copies, load, iters, max_before


def zipf_loads(rng, E, total, s):
    w = 1.0 / np.arange(1, E + 1) ** s
    w = w[rng.permutation(E)]
    return rng.multinomial(total, w / w.sum()).astype(np.int32)


@pytest.mark.parametrize("R,M,S", [(2, 2, 1), (4, 2, 2), (8, 2, 2), (5, 4, 3), (16, 1, 4),
                                   (3, 3, 0), (64, 2, 2)])
@pytest.mark.parametrize("min_tokens", [0, 3])
def test_pick_order_then_rank_side_equals_the_greedy(R, M, S, min_tokens):
    E = R * M
    rng = np.random.default_rng(R * 100 + M * 10 + S + min_tokens)
    for trial in range(8):
        load_e = zipf_loads(rng, E, int(rng.integers(1, 40 * R)), float(rng.uniform(0.5, 2.5)))
        pl = oracle.plan(load_e, R, S, min_tokens)
        slot_expert, copies, load, iters, max_before = plan_by_picks(load_e, R, S, min_tokens)
        assert list(pl.slot_expert) == slot_expert
        assert list(pl.n_copies) == copies
        assert list(pl.rank_load) == load
        assert int(pl.stats[0]) == iters and int(pl.stats[1]) == max_before


def test_layouts_where_copies_outnumber_pairs():
    for load_e, R, S in [([3, 0], 2, 3), ([3, 1, 0, 0, 0, 0, 0, 0], 4, 4),
                         ([2, 1, 0, 0, 0, 0], 3, 2)]:
        load_e = np.array(load_e, dtype=np.int32)
        pl = oracle.plan(load_e, R, S)
        slot_expert, copies, load, iters, _ = plan_by_picks(load_e, R, S)
        assert list(pl.slot_expert) == slot_expert and list(pl.n_copies) == copies
        assert list(pl.rank_load) == load and int(pl.stats[0]) == iters
        assert any(c > L > 0 for c, L in zip(copies, load_e))

"""The routing half of the path at the size limits of the C ABI: R = 128
ranks, E = 256 experts, K = 32, S = 2, and Q = R*T*K = 2^30 - 16384 pairs, just
below the limit (the look-back counts and the dispatch rows are 30-bit and
int32). The oracle cannot walk a billion pairs in a test, so the results are
checked on the device by properties that fix them completely given the plan:

* the counts equal a plain histogram (torch.bincount);
* the plan's quotas of each expert sum to its load, and the slot offsets are
  their running sum;
* dest_row is a permutation of [0, Q); every pair lands on a copy of its own
  expert; every slot receives exactly its quota;
* inside a slot the rows follow the global pair order (the prefix fill is
  stable), which with the counts per slot determines every row.

The ids are not drawn by the gate: token n routes to experts (h(n) + k) mod E,
k = 0..K-1, with h(n) skewed toward a few hot bases (a torch generator), so
every row holds K distinct experts and some experts are far above the mean.
"""
import pytest
import torch

import token_rerouting_b200 as ue
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

R, E, K, S = 128, 256, 32, 2
T = ((1 << 30) - (1 << 14)) // (R * K)
M, G, P = E // R, R * S, R * (E // R + S)


def test_routing_at_the_size_limits():
    gh.ensure_built()
    dev = torch.device("cuda", 0)
    N, Q = R * T, R * T * K
    assert Q < (1 << 30) and Q >= (1 << 30) - (1 << 14)
    cfg = ue.make_config(R, T, E, K, S, 8)
    ctx = ue.ue_init(cfg, 0)
    try:
        g = torch.Generator(device=dev).manual_seed(11)
        # skewed bases: half the tokens start at one of 4 hot bases
        hot = torch.tensor([3, 77, 140, 201], device=dev)
        h = torch.randint(0, E, (N,), device=dev, generator=g)
        pick_hot = torch.rand((N,), device=dev, generator=g) < 0.5
        h = torch.where(pick_hot, hot[torch.randint(0, 4, (N,), device=dev, generator=g)], h)
        idx = ((h[:, None] + torch.arange(K, device=dev)[None, :]) % E).to(torch.int32)
        del h, pick_hot
        load_re = torch.empty((R, E), dtype=torch.int32, device=dev)
        load_e = torch.empty(E, dtype=torch.int32, device=dev)
        ue.ue_count(ctx, idx, load_re, load_e)
        ref = torch.bincount(idx.view(-1).long(), minlength=E)
        assert torch.equal(load_e.long(), ref)
        assert int(load_re.long().sum()) == Q

        arrs = dict(slot_expert=torch.empty(G, dtype=torch.int32, device=dev),
                    n_copies=torch.empty(E, dtype=torch.int32, device=dev),
                    slot_quota=torch.empty(P, dtype=torch.int32, device=dev),
                    slot_offset=torch.empty(P + 1, dtype=torch.int32, device=dev),
                    rank_load=torch.empty(R, dtype=torch.int32, device=dev),
                    stats=torch.empty(4, dtype=torch.int32, device=dev))
        plan = ue.placement(arrs["slot_expert"], arrs["n_copies"], arrs["slot_quota"],
                            arrs["slot_offset"], arrs["rank_load"], arrs["stats"])
        ue.ue_plan(ctx, load_e, plan)
        phys = torch.empty((N, K), dtype=torch.int32, device=dev)
        dest = torch.empty((N, K), dtype=torch.int32, device=dev)
        ue.ue_reroute(ctx, idx, plan, phys, dest)
        assert ue.ue_get_error(ctx) == ue.UE_OK

        # the plan: quotas per expert sum to its load; offsets are their scan
        p = torch.arange(P, device=dev)
        r_of, l_of = p // (M + S), p % (M + S)
        se = arrs["slot_expert"].long()
        owner = torch.where(l_of < M, r_of * M + l_of,
                            se[(r_of * S + (l_of - M)).clamp(0, G - 1)])
        owner = torch.where((l_of >= M) & (owner < 0), torch.full_like(owner, -1), owner)
        quota = arrs["slot_quota"].long()
        used = owner >= 0
        per_e = torch.zeros(E, dtype=torch.long, device=dev).index_add_(0, owner[used], quota[used])
        assert torch.equal(per_e, ref)
        assert int(quota[~used].abs().sum()) == 0
        offs = torch.cat([torch.zeros(1, dtype=torch.long, device=dev), quota.cumsum(0)])
        assert torch.equal(arrs["slot_offset"].long(), offs)
        stats = arrs["stats"].cpu().tolist()
        assert stats[0] > 0  # the skew makes the greedy replicate

        # the reroute, checked in chunks of 2^26 pairs to bound the memory
        CH = 1 << 26
        idx_f, phys_f, dest_f = idx.view(-1), phys.view(-1), dest.view(-1)
        counts = torch.zeros(P, dtype=torch.long, device=dev)
        for a in range(0, Q, CH):
            ph = phys_f[a:a + CH].long()
            assert bool((ph >= 0).all()) and bool((ph < P).all())
            assert torch.equal(owner[ph], idx_f[a:a + CH].long())  # a copy of its own expert
            counts += torch.bincount(ph, minlength=P)
        assert torch.equal(counts, quota)                           # exactly its quota
        del idx, idx_f
        rows_sorted, order = torch.sort(dest_f)
        for a in range(0, Q, CH):                                    # a permutation of [0, Q)
            n = min(CH, Q - a)
            assert torch.equal(rows_sorted[a:a + n],
                               torch.arange(a, a + n, device=dev, dtype=torch.int32))
        del rows_sorted
        # rows of a slot follow the pair order, and each slot starts at its offset
        first_row = torch.full((P,), -1, dtype=torch.long, device=dev)
        prev_slot, prev_pair = None, None
        for a in range(0, Q, CH):
            n = min(CH, Q - a)
            o = order[a:a + n]
            sl = phys_f[o].long()
            if prev_slot is not None:
                sl_ext = torch.cat([prev_slot.view(1), sl])
                o_ext = torch.cat([prev_pair.view(1), o])
            else:
                sl_ext, o_ext = sl, o
            same = sl_ext[1:] == sl_ext[:-1]
            assert bool((~same | (o_ext[1:] > o_ext[:-1])).all())
            starts = torch.ones(n, dtype=torch.bool, device=dev)
            if prev_slot is not None:
                starts = ~same
            else:
                starts[1:] = ~same
            pos = torch.nonzero(starts).view(-1)
            first_row[sl[pos]] = pos + a
            prev_slot, prev_pair = sl[-1], o[-1]
        nonempty = quota > 0
        assert torch.equal(first_row[nonempty], offs[:-1][nonempty])
    finally:
        ue.ue_destroy(ctx)

"""The non-stationary sweep: 48 layers x 8 microbatches of the Qwen3-shaped
layer (R=64, 4096 tokens per rank, E=128, K=8, S=2, d=4096), Zipf exponent
and hot set redrawn per instance, with a uniform instance (0,0) and a
30%-single-expert instance (0,1). The whole path is captured once as a CUDA
graph over fixed buffers; each instance's logits are staged into the input
buffer and the graph is replayed.

Every instance's routing (top-k ids, counts, every plan array, phys_slot,
dest_row) is compared with the oracle's, byte for byte, through a SHA-256
digest the oracle wrote for that instance (tests/golden/sweep_digests.py);
on a mismatch the oracle is run on the instance to name the array that
differs. Every instance's gate weights are compared with the oracle's on a
sample of rows, and every instance is also checked on the device by
properties (dest_row is a permutation of the pairs; each slot receives
exactly its quota; each pair lands on a copy of its own expert; rank loads
sum to the pairs). Eight instances, the two special ones included, are also
compared with the oracle element by element on the routing, on sampled
dispatch rows, and on the combine with independent expert outputs (every
token under the greedy plan, a token sample under the capacity planner).

The sweep runs twice: with the path's greedy plan, and with the capacity
planner at the pages' defaults ("UltraEP" README, "Performance Tuning /
Replication planning": eps 0.01, early stop at 1.0, at least 1024 pairs per
replica), whose every instance is also checked against its own guarantees
(rank loads within the chosen capacity C(k) = floor(k Q / (100 R)), every
replica at least 1024 pairs).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import gpu_helpers as gh
from tests.routing_digest import flatten_oracle, routing_digest

DIGESTS = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                       "sweep_digests.json")

pytestmark = pytest.mark.gpu


def slot_owner(L, dev):
    """Expert held by every physical slot (-1 for an empty redundant slot)."""
    M, S, R = L.M, L.S, L.R
    p = torch.arange(L.P, device=dev)
    r, l = p // (M + S), p % (M + S)
    owner = torch.where(l < M, r * M + l, torch.full_like(p, -1))
    if L.G > 0:
        g = r * S + (l - M)
        rep = L.slot_expert[: L.G].long()[g.clamp(0, L.G - 1)]
        owner = torch.where(l < M, owner, rep)
    return owner


@pytest.mark.parametrize("planner", ["greedy", "bisect"])
def test_sweep_graph_captured(planner):
    import token_rerouting_b200 as ue
    w = synth.WORKLOADS["sweep_48x8_r64_e128"]
    L = gh.make_layer(w.R, w.T, w.E, w.K, w.S, w.d)
    dev = L.device
    opts = ue.plan_opts(ue.UE_SOLVER_BISECT) if planner == "bisect" else None

    def run_once(st):
        L.gate_count(st)
        if opts is None:
            L.plan_reroute(st)
        else:
            L.plan_ex(opts, st)
            L.reroute(st)
        L.permute(st)
        L.combine(stream=st)

    with open(DIGESTS) as f:
        digests = json.load(f)["digests"][planner]
    assert len(digests) == w.layers * w.microbatches

    def oracle_path(logits):
        if opts is None:
            return oracle.run_path(logits, w.R, w.T, w.S, w.K)
        idx, wts = oracle.gate_topk(logits, w.K)
        load_re, load_e = oracle.count(idx, w.R, w.T, w.E)
        pl = oracle.plan_bisect(load_e, w.R, w.S)
        phys, dest = oracle.reroute(idx, w.R, w.E, w.S, pl)
        return dict(idx=idx, w=wts, load_re=load_re, load_e=load_e, plan=pl,
                    phys_slot=phys, dest_row=dest)

    try:
        hidden = synth.hidden(w)
        sigma = synth.expert_output_rows(w)
        L.hidden.copy_(gh.bf16_to_device(hidden, dev))
        L.logits.copy_(torch.from_numpy(synth.logits(w, 0, 0)))
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            run_once(s)
        torch.cuda.current_stream(dev).wait_stream(s)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            run_once(s)
        torch.cuda.synchronize(dev)

        rng = np.random.default_rng(5)
        others = [(int(x) // w.microbatches, int(x) % w.microbatches)
                  for x in rng.choice(np.arange(2, w.layers * w.microbatches), 6, replace=False)]
        exact = {(0, 0), (0, 1), *others}
        ar = torch.arange(w.Q, device=dev, dtype=torch.int32)
        iters, skew_before, skew_after = [], [], []
        for layer in range(w.layers):
            for mb in range(w.microbatches):
                logits = synth.logits(w, layer, mb)
                L.logits.copy_(torch.from_numpy(logits))
                graph.replay()
                torch.cuda.synchronize(dev)
                # properties, on the device
                dest = L.dest_row.flatten()
                assert torch.equal(torch.sort(dest).values, ar), (layer, mb)
                phys = L.phys_slot.flatten().long()
                counts = torch.bincount(phys, minlength=L.P)
                assert torch.equal(counts.int(), L.slot_quota), (layer, mb)
                owner = slot_owner(L, dev)
                assert torch.equal(owner[phys], L.idx.flatten().long()), (layer, mb)
                assert int(L.rank_load.long().sum()) == w.Q
                st = L.stats.cpu().numpy()
                iters.append(int(st[0]))
                skew_before.append(st[1] / (w.Q / w.R))
                skew_after.append(st[2] / (w.Q / w.R))
                if opts is not None:
                    cap = int(st[3]) * w.Q // (100 * w.R)
                    assert int(L.rank_load.max()) <= cap, (layer, mb)
                    used = L.slot_expert[: w.G] >= 0
                    if bool(used.any()):
                        rep_q = L.slot_quota.view(w.R, w.M + w.S)[:, w.M:].flatten()[used]
                        assert int(rep_q.min()) >= 1024, (layer, mb)
                # every instance: the routing against the oracle's digest
                g = gh.routing_results(L)
                inst = layer * w.microbatches + mb
                if routing_digest(g) != digests[inst] or (layer, mb) in exact:
                    o = oracle_path(logits)
                    gh.assert_routing_equal(g, o)
                    assert routing_digest(flatten_oracle(o)) == digests[inst], (
                        "stored digest differs from the oracle's routing", layer, mb)
                # every instance: gate weights on a row sample
                wrows = np.sort(rng.choice(w.N, 1024, replace=False))
                _, w_or = oracle.gate_topk(logits[wrows], w.K)
                gh.assert_weights_close(g["w"][wrows], w_or)
                if (layer, mb) in exact:
                    rows = np.sort(np.concatenate([
                        rng.choice(w.Q, 16384, replace=False),
                        o["plan"].slot_offset[np.nonzero(o["plan"].slot_quota)[0]]]))
                    rows = np.unique(rows)
                    got = gh.bf16_to_host_u16(L.dispatch[torch.from_numpy(rows).to(dev)])
                    np.testing.assert_array_equal(
                        got, oracle.permute_rows(hidden, w.K, o["dest_row"], rows))
                    # combine with independent expert outputs
                    gh.expert_outputs_on_device(L, hidden, sigma)
                    L.combine()
                    toks = (None if opts is None
                            else np.sort(rng.choice(w.N, 16384, replace=False)))
                    gh.assert_combine_all_tokens(L, hidden, sigma, w.K, o["dest_row"], o["w"],
                                                 tokens=toks)
        assert L.error() == 0
        # the sweep spans balanced and heavily skewed instances
        assert min(skew_before) < 1.1 and max(skew_before) > 2.0
        if opts is not None:
            # the capacity planner brings every instance to within a few
            # grid steps of the mean
            assert max(skew_after) < 1.1, max(skew_after)
        assert len(iters) == w.layers * w.microbatches
    finally:
        L.close()
